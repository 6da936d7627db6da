// Split-K combine, value bound E_val, block-ranking consistency check and the
// rung 3 / rung 4 decisions; and the combine of the dense fallback.
//
// Runtime-Certified Bounded-Error Quantized Attention, Methodology §2
// (E_val = sum over INT4-valued blocks of attention mass times eta_b) and §3
// (rank-consistency check: the INT8 ranking of the promoted blocks is compared
// with their FP16 ranking, a mismatch sends the head to dense attention;
// rung 4 recomputes the whole layer densely).
//
// Readings used: the check compares the ordered top-min(rank_r, |P|) lists of
// promoted blocks by INT8 and by FP16 block log-mass (ties to the lower block
// index); rung 3 also fires when E_key stayed above eps_key after widening or
// when E_val > eps_val; rung 4 fires when at least need_dense =
// ceil(layer_dense_frac * n_q_heads) heads of a (layer, batch row) took rung 3.
#include "cqa_internal.cuh"

namespace cqa {

namespace {

struct KI {
  float k;
  int i;
};

// (key descending, index ascending): true when a comes before b
__device__ __forceinline__ bool before(KI a, KI b) { return a.k > b.k || (a.k == b.k && a.i < b.i); }

// Best promoted block strictly after `prev` in the ranking order (warp-wide).
__device__ KI next_best(const float* key, const uint8_t* bf, int nb, KI prev, int lane) {
  KI best{-INFINITY, 0x7fffffff};
  for (int j = lane; j < nb; j += 32) {
    if (!(bf[j] & BF_KEY)) continue;
    const KI c{key[j], j};
    if (before(prev, c) && before(c, best)) best = c;
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
    KI o;
    o.k = __shfl_xor_sync(0xffffffffu, best.k, m);
    o.i = __shfl_xor_sync(0xffffffffu, best.i, m);
    if (before(o, best)) best = o;
  }
  return best;
}

template <int D, int G>
__global__ void combine_kernel(DecodeShape sh, cqa_thresholds th, int need_dense, Scratch sc,
                               float* __restrict__ out, float* __restrict__ e_key,
                               float* __restrict__ e_val, uint8_t* __restrict__ rung) {
  constexpr int CPL = D / 32;  // channels per lane
  __shared__ int n3;
  extern __shared__ uint8_t r3[];  // [Hq]
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
  const bool naive = th.naive != 0;
  if (threadIdx.x == 0) n3 = 0;
  __syncthreads();

  for (int h = warp; h < sh.Hq; h += nwarp) {
    const int g = h / G, hh = h - g * G;
    const int unit = b * sh.Hkv + g;
    const size_t row = (size_t)b * sh.Hq + h;
    float M = -INFINITY;
    for (int c = 0; c < sh.nchunks; ++c)
      M = fmaxf(M, sc.part_s[(((size_t)unit * sc.max_chunks + c) * G + hh) * 3]);
    float L = 0.f, E = 0.f, o[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) o[k] = 0.f;
    for (int c = 0; c < sh.nchunks; ++c) {
      const size_t pi = ((size_t)unit * sc.max_chunks + c) * G + hh;
      const float mc = sc.part_s[pi * 3];
      const float w = mc == -INFINITY ? 0.f : expf(mc - M);
      L += sc.part_s[pi * 3 + 1] * w;
      E += sc.part_s[pi * 3 + 2] * w;
#pragma unroll
      for (int k = 0; k < CPL; ++k) o[k] += sc.part_o[pi * D + lane + 32 * k] * w;
    }
    const float inv = 1.f / L;
#pragma unroll
    for (int k = 0; k < CPL; ++k) out[row * D + lane + 32 * k] = o[k] * inv;
    const float ev = E * inv;

    uint8_t hf = sc.hflags[row];
    if (!naive) {
      const uint8_t* bf = sc.bflags + (size_t)unit * sh.nbm;
      const float* e8 = sc.ell8 + row * sh.nbm;
      const float* e16 = sc.ell16 + row * sh.nbm;
      int np = 0;
      for (int j = lane; j < sh.nb; j += 32) np += (bf[j] & BF_KEY) ? 1 : 0;
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) np += __shfl_xor_sync(0xffffffffu, np, m);
      const int r = min(th.rank_r, np);
      KI p8{INFINITY, -1}, p16{INFINITY, -1};
      bool fail = false;
      for (int k = 0; k < r && !fail; ++k) {
        p8 = next_best(e8, bf, sh.nb, p8, lane);
        p16 = next_best(e16, bf, sh.nb, p16, lane);
        fail = p8.i != p16.i;
      }
      if (fail) hf |= HF_RANKFAIL;
      if (ev > th.eps_val) hf |= HF_VALFAIL;
    }
    const bool is3 = !naive && (hf & (HF_KEYFAIL | HF_RANKFAIL | HF_VALFAIL));
    if (lane == 0) {
      sc.hflags[row] = hf;
      e_key[row] = sc.ekey[row];
      e_val[row] = ev;
      rung[row] = (hf & HF_VALUE) ? 2 : ((hf & HF_WIDENED) ? 1 : 0);
      r3[h] = is3 ? 1 : 0;
      if (is3) atomicAdd(&n3, 1);
    }
  }
  __syncthreads();
  const bool layer = !naive && n3 >= need_dense;
  for (int h = threadIdx.x; h < sh.Hq; h += blockDim.x) {
    const size_t row = (size_t)b * sh.Hq + h;
    const uint8_t dv = layer ? 4 : (r3[h] ? 3 : 0);
    sc.dense[row] = dv;
    if (dv) rung[row] = dv;
  }
}

// One warp per (batch row, query head); only dense heads are written.
template <int D, int G>
__global__ void dense_combine_kernel(DecodeShape sh, Scratch sc, int all_heads,
                                     float* __restrict__ out, float* __restrict__ e_key,
                                     float* __restrict__ e_val, uint8_t* __restrict__ rung) {
  constexpr int CPL = D / 32;
  const int row = blockIdx.x;  // b * Hq + h
  const int lane = threadIdx.x;
  const int b = row / sh.Hq, h = row - b * sh.Hq;
  const uint8_t dv = all_heads ? 4 : sc.dense[row];
  if (dv == 0) return;
  const int g = h / G, hh = h - g * G;
  const int unit = b * sh.Hkv + g;
  float M = -INFINITY;
  for (int c = 0; c < sh.nchunks; ++c)
    M = fmaxf(M, sc.part_s[(((size_t)unit * sc.max_chunks + c) * G + hh) * 3]);
  float L = 0.f, o[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) o[k] = 0.f;
  for (int c = 0; c < sh.nchunks; ++c) {
    const size_t pi = ((size_t)unit * sc.max_chunks + c) * G + hh;
    const float mc = sc.part_s[pi * 3];
    const float w = mc == -INFINITY ? 0.f : expf(mc - M);
    L += sc.part_s[pi * 3 + 1] * w;
#pragma unroll
    for (int k = 0; k < CPL; ++k) o[k] += sc.part_o[pi * D + lane + 32 * k] * w;
  }
  const float inv = 1.f / L;
#pragma unroll
  for (int k = 0; k < CPL; ++k) out[(size_t)row * D + lane + 32 * k] = o[k] * inv;
  if (!all_heads && lane == 0) {
    e_key[row] = 0.f;
    e_val[row] = 0.f;
    rung[row] = dv;
  }
}

template <int D, int G>
cudaError_t combine_t(const DecodeShape& sh, const cqa_thresholds& th, int need_dense,
                      const Scratch& sc, float* out, float* e_key, float* e_val, uint8_t* rung,
                      cudaStream_t s) {
  const int threads = 32 * (sh.Hq < 32 ? sh.Hq : 32);
  combine_kernel<D, G><<<sh.B, threads, sh.Hq, s>>>(sh, th, need_dense, sc, out, e_key, e_val,
                                                    rung);
  return cudaGetLastError();
}

template <int D, int G>
cudaError_t dense_combine_t(const DecodeShape& sh, const Scratch& sc, int all_heads, float* out,
                            float* e_key, float* e_val, uint8_t* rung, cudaStream_t s) {
  dense_combine_kernel<D, G><<<sh.B * sh.Hq, 32, 0, s>>>(sh, sc, all_heads, out, e_key, e_val,
                                                         rung);
  return cudaGetLastError();
}

}  // namespace

#define CQA_DISPATCH_DG(FN, ...)                                   \
  do {                                                             \
    if (sh.d == 128) {                                             \
      switch (sh.G) {                                              \
        case 1: return FN<128, 1>(__VA_ARGS__);                    \
        case 2: return FN<128, 2>(__VA_ARGS__);                    \
        case 4: return FN<128, 4>(__VA_ARGS__);                    \
        case 8: return FN<128, 8>(__VA_ARGS__);                    \
      }                                                            \
    } else {                                                       \
      switch (sh.G) {                                              \
        case 1: return FN<64, 1>(__VA_ARGS__);                     \
        case 2: return FN<64, 2>(__VA_ARGS__);                     \
        case 4: return FN<64, 4>(__VA_ARGS__);                     \
      }                                                            \
    }                                                              \
    return cudaErrorInvalidValue;                                  \
  } while (0)

cudaError_t launch_combine(const DecodeShape& sh, const cqa_thresholds& th, int need_dense,
                           const Scratch& sc, float* out, float* e_key, float* e_val,
                           uint8_t* rung, cudaStream_t s) {
  CQA_DISPATCH_DG(combine_t, sh, th, need_dense, sc, out, e_key, e_val, rung, s);
}

cudaError_t launch_dense_combine(const DecodeShape& sh, const Scratch& sc, int all_heads,
                                 float* out, float* e_key, float* e_val, uint8_t* rung,
                                 cudaStream_t s) {
  CQA_DISPATCH_DG(dense_combine_t, sh, sc, all_heads, out, e_key, e_val, rung, s);
}

}  // namespace cqa
