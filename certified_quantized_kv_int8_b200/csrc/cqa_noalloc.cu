// Exact decode attention over caller-provided FP16 keys and values that
// allocates no memory at all: its split-K scratch lives in a fixed
// file-scope device array.
//
// Who needs this: callers that cannot call cudaMalloc.  Typical cases are
// hosts that hand a fixed memory budget to several libraries and own the only
// device allocator (memory a library allocated on its own would be memory the
// host already promised elsewhere), and latency-critical paths where
// cudaMalloc/cudaFree may synchronise the device.  Such callers still pass
// their own inputs and outputs; the only memory this entry point needs beyond
// them is the scratch array below.
//
// Shapes: head_dim 64 or 128, n_q_heads / n_kv_heads in {1, 2, 4, 8} (8 only
// at head_dim 128), batch * n_kv_heads <= 65535, and the partials of one
// chunk per kv head within the array's 4 MiB.
//
// The paper has no counterpart of this entry point; it is a deployment
// convenience of this library.
#include <mutex>

#include "cqa_internal.cuh"

namespace cqa {

namespace {

constexpr int NA_THREADS = 256;

// Split-K partials: [units][chunks][G][D + 3] floats (m, l, then o[D]).
// Every partial is written before it is read, so nothing needs clearing.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CQA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device, set up once per device.
std::mutex g_mu;
void* g_scratch_addr[256];
bool g_scratch_ready[256];

__device__ __forceinline__ float na_warp_max(float x) {
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ float na_warp_sum(float x) {
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// grid (chunks, B*Hkv).  CTA: the G query heads of one kv head over a chunk
// of 64-token blocks; token loads are guarded by T, so K and V need no padding.
template <int D, int G>
__global__ void __launch_bounds__(NA_THREADS)
    noalloc_dense_kernel(const __half* __restrict__ q, const __half* __restrict__ k,
                         const __half* __restrict__ v, int Hq, int Hkv, int T, int chunk_blocks,
                         int nchunks, float sigma, float* __restrict__ scratch) {
  constexpr int LPR = D / 8;          // threads per token row, 8 channels each
  constexpr int RPC = NA_THREADS / LPR;
  constexpr int NPASS = BLK / RPC;
  __shared__ float kpart[G][BLK][LPR + 1];
  __shared__ float pp[G][BLK];
  __shared__ float red[RPC][D];
  __shared__ float sm[G], sl[G], salpha[G];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.y, chunk = blockIdx.x;
  const int b = unit / Hkv, g = unit - b * Hkv;
  const size_t hrow0 = (size_t)b * Hq + (size_t)g * G;
  const __half* ku = k + (size_t)unit * T * D;
  const __half* vu = v + (size_t)unit * T * D;
  const int nblk = (T + BLK - 1) / BLK;
  const int j0 = chunk * chunk_blocks, j1 = min(nblk, j0 + chunk_blocks);
  const int row = tid / LPR, cl = tid - row * LPR;

  float2 qr[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 qv = *reinterpret_cast<const uint4*>(q + (hrow0 + h) * D + cl * 8);
    const __half2* qh = reinterpret_cast<const __half2*>(&qv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(qh[i]);
      qr[h][i] = make_float2(f.x * sigma, f.y * sigma);
    }
  }
  float2 acc[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[h][i] = make_float2(0.f, 0.f);
  if (tid < G) {
    sm[tid] = -INFINITY;
    sl[tid] = 0.f;
  }

  for (int j = j0; j < j1; ++j) {
    const int tok0 = j * BLK;
    const int ntok = min(BLK, T - tok0);
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
      const int tt = p * RPC + row;
      float2 kf[4];
      if (tt < ntok) {
        const uint4 kv = *reinterpret_cast<const uint4*>(ku + (size_t)(tok0 + tt) * D + cl * 8);
        const __half2* kh = reinterpret_cast<const __half2*>(&kv);
#pragma unroll
        for (int i = 0; i < 4; ++i) kf[i] = __half22float2(kh[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) kf[i] = make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) a = __ffma2_rn(qr[h][i], kf[i], a);
        kpart[h][tt][cl] = a.x + a.y;
      }
    }
    __syncthreads();
    if (warp < G) {
      const int h = warp;
      float x[2];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int tt = lane + 32 * s;
        float acc_l = 0.f;
#pragma unroll
        for (int i = 0; i < LPR; ++i) acc_l += kpart[h][tt][i];
        x[s] = tt < ntok ? acc_l : -INFINITY;
      }
      const float mb = na_warp_max(fmaxf(x[0], x[1]));
      const float mold = sm[h];
      const float mnew = fmaxf(mold, mb);
      const float alpha = mold == -INFINITY ? 0.f : expf(mold - mnew);
      const float p0 = expf(x[0] - mnew), p1 = expf(x[1] - mnew);
      pp[h][lane] = p0;
      pp[h][lane + 32] = p1;
      const float sb = na_warp_sum(p0 + p1);
      if (lane == 0) {
        sl[h] = sl[h] * alpha + sb;
        sm[h] = mnew;
        salpha[h] = alpha;
      }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float al = salpha[h];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[h][i].x *= al;
        acc[h][i].y *= al;
      }
    }
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
      const int tt = p * RPC + row;
      if (tt >= ntok) continue;
      const uint4 vv = *reinterpret_cast<const uint4*>(vu + (size_t)(tok0 + tt) * D + cl * 8);
      const __half2* vh = reinterpret_cast<const __half2*>(&vv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 vf = __half22float2(vh[i]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float w = pp[h][tt];
          acc[h][i] = __ffma2_rn(make_float2(w, w), vf, acc[h][i]);
        }
      }
    }
    __syncthreads();
  }

  float* part = scratch + ((size_t)unit * nchunks + chunk) * G * (D + 3);
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      red[row][cl * 8 + 2 * i] = acc[h][i].x;
      red[row][cl * 8 + 2 * i + 1] = acc[h][i].y;
    }
    __syncthreads();
    for (int c = tid; c < D; c += NA_THREADS) {
      float s = 0.f;
      for (int r = 0; r < RPC; ++r) s += red[r][c];
      part[h * (D + 3) + 3 + c] = s;
    }
    __syncthreads();
  }
  if (tid < G) {
    part[tid * (D + 3) + 0] = sm[tid];
    part[tid * (D + 3) + 1] = sl[tid];
    part[tid * (D + 3) + 2] = 0.f;
  }
}

// one warp per (batch row, query head)
template <int D, int G>
__global__ void noalloc_combine_kernel(int Hq, int Hkv, int nchunks,
                                       const float* __restrict__ scratch,
                                       float* __restrict__ out) {
  constexpr int CPL = D / 32;
  const int rowi = blockIdx.x, lane = threadIdx.x;
  const int b = rowi / Hq, h = rowi - b * Hq;
  const int g = h / G, hh = h - g * G;
  const int unit = b * Hkv + g;
  float M = -INFINITY;
  for (int c = 0; c < nchunks; ++c)
    M = fmaxf(M, scratch[(((size_t)unit * nchunks + c) * G + hh) * (D + 3)]);
  float L = 0.f, o[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) o[i] = 0.f;
  for (int c = 0; c < nchunks; ++c) {
    const float* part = scratch + (((size_t)unit * nchunks + c) * G + hh) * (D + 3);
    const float mc = part[0];
    const float w = mc == -INFINITY ? 0.f : expf(mc - M);
    L += part[1] * w;
#pragma unroll
    for (int i = 0; i < CPL; ++i) o[i] += part[3 + lane + 32 * i] * w;
  }
  const float inv = 1.f / L;
#pragma unroll
  for (int i = 0; i < CPL; ++i) out[(size_t)rowi * D + lane + 32 * i] = o[i] * inv;
}

template <int D, int G>
cudaError_t launch_noalloc(const __half* q, const __half* k, const __half* v, int B, int Hq,
                           int Hkv, int T, int chunk_blocks, int nchunks, float* scratch,
                           float* out, cudaStream_t s) {
  const float sigma = (float)(1.0 / sqrt((double)D));
  noalloc_dense_kernel<D, G><<<dim3(nchunks, B * Hkv), NA_THREADS, 0, s>>>(
      q, k, v, Hq, Hkv, T, chunk_blocks, nchunks, sigma, scratch);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  noalloc_combine_kernel<D, G><<<B * Hq, 32, 0, s>>>(Hq, Hkv, nchunks, scratch, out);
  return cudaGetLastError();
}

}  // namespace

}  // namespace cqa

extern "C" int cqa_dense_attention_noalloc(const void* q_fp16, const void* k_fp16,
                                           const void* v_fp16, int batch, int n_q_heads,
                                           int n_kv_heads, int head_dim, int n_tokens,
                                           float* out, void* stream) {
  using namespace cqa;
  if (!q_fp16 || !k_fp16 || !v_fp16 || !out) return CQA_ERR_INVALID_ARG;
  if (((uintptr_t)q_fp16 | (uintptr_t)k_fp16 | (uintptr_t)v_fp16 | (uintptr_t)out) & 15u)
    return CQA_ERR_INVALID_ARG;
  if (batch < 1 || n_q_heads < 1 || n_kv_heads < 1 || n_tokens < 1) return CQA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return CQA_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads) return CQA_ERR_INVALID_ARG;
  const int G = n_q_heads / n_kv_heads;
  if (!(G == 1 || G == 2 || G == 4 || G == 8) || (head_dim == 64 && G == 8))
    return CQA_ERR_INVALID_ARG;

  // split-K chunking: about four CTAs per SM over all units, limited by the scratch size
  const long long units = (long long)batch * n_kv_heads;
  const long long nblk = (n_tokens + BLK - 1) / BLK;
  const size_t per_part = (size_t)G * (head_dim + 3) * sizeof(float);
  const long long cap_parts = (long long)(CQA_NOALLOC_SCRATCH_BYTES / per_part);
  if (units > cap_parts) return CQA_ERR_CAPACITY;  // even one chunk per unit does not fit
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
    cudaGetLastError();
    return CQA_ERR_CUDA;
  }
  long long per_unit = ((long long)sms * 4 + units - 1) / units;
  if (per_unit > cap_parts / units) per_unit = cap_parts / units;
  if (per_unit < 1) per_unit = 1;
  const int chunk_blocks = (int)((nblk + per_unit - 1) / per_unit);
  const int nchunks = (int)((nblk + chunk_blocks - 1) / chunk_blocks);
  if ((size_t)units * nchunks * per_part > CQA_NOALLOC_SCRATCH_BYTES) return CQA_ERR_CAPACITY;
  if (units > 65535) return CQA_ERR_CAPACITY;

  // one-time set-up per device: the host-side name of the array is not a
  // device address, so look the address up with this device current
  if (dev < 0 || dev >= 256) return CQA_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ready[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return CQA_ERR_CUDA;
      }
      g_scratch_addr[dev] = p;
      g_scratch_ready[dev] = true;
    }
    scratch = g_scratch_addr[dev];
  }

  const __half* q = (const __half*)q_fp16;
  const __half* k = (const __half*)k_fp16;
  const __half* v = (const __half*)v_fp16;
  float* sc = (float*)scratch;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaErrorInvalidValue;
  if (head_dim == 128) {
    switch (G) {
      case 1: e = launch_noalloc<128, 1>(q, k, v, batch, n_q_heads, n_kv_heads, n_tokens, chunk_blocks, nchunks, sc, out, s); break;
      case 2: e = launch_noalloc<128, 2>(q, k, v, batch, n_q_heads, n_kv_heads, n_tokens, chunk_blocks, nchunks, sc, out, s); break;
      case 4: e = launch_noalloc<128, 4>(q, k, v, batch, n_q_heads, n_kv_heads, n_tokens, chunk_blocks, nchunks, sc, out, s); break;
      case 8: e = launch_noalloc<128, 8>(q, k, v, batch, n_q_heads, n_kv_heads, n_tokens, chunk_blocks, nchunks, sc, out, s); break;
    }
  } else {
    switch (G) {
      case 1: e = launch_noalloc<64, 1>(q, k, v, batch, n_q_heads, n_kv_heads, n_tokens, chunk_blocks, nchunks, sc, out, s); break;
      case 2: e = launch_noalloc<64, 2>(q, k, v, batch, n_q_heads, n_kv_heads, n_tokens, chunk_blocks, nchunks, sc, out, s); break;
      case 4: e = launch_noalloc<64, 4>(q, k, v, batch, n_q_heads, n_kv_heads, n_tokens, chunk_blocks, nchunks, sc, out, s); break;
    }
  }
  return e == cudaSuccess ? CQA_OK : CQA_ERR_CUDA;
}
