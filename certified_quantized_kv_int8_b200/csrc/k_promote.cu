// Promotion: FP16 keys of the promoted blocks, read straight from the pinned,
// device-mapped Tier 2 over the host link, turned into exact logits that
// replace the blocks' INT8 logits in place, plus each promoted block's FP16
// log-mass ell16_b for the rank-consistency check.  A second mode computes the
// exact logits of the not-promoted blocks for heads that fall back to dense
// attention.
//
// Runtime-Certified Bounded-Error Quantized Attention, Methodology §3 (the
// top-K* blocks get FP16 keys paged from Tier 2; the rank check compares the
// INT8 and FP16 block rankings of the promoted blocks; rungs 3-4 recompute
// heads or layers from the FP16 originals) and §1 (Tier 2 in pinned host RAM).
//
// Reading Tier 2 directly, the kernel is bound by the host link: it streams
// 16 KiB of keys per block and kv head and writes 1 KiB of logits.  Each CTA
// keeps two blocks of keys in flight (the next block's loads are issued before
// the current block is reduced) so the link stays busy.  When the library has
// staged the layer's keys in device memory ahead of time (a whole-layer copy
// by the copy engine, see cqa_set_key_prefetch), staged blocks are read from
// HBM instead; the values are identical, only the path differs.
#include "cqa_internal.cuh"

namespace cqa {

namespace {

constexpr int THREADS = 256;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// MODE 0: blocks with BF_KEY, every head, write ell16.
// MODE 1: blocks without BF_KEY of units holding a dense head, dense heads only.
template <int D, int G, int MODE>
__global__ void __launch_bounds__(THREADS) promote_kernel(Tier1 t, Strides st, int unit0,
                                                          DecodeShape sh,
                                                          const __half* __restrict__ q,
                                                          Scratch sc,
                                                          const __half* __restrict__ kstage,
                                                          int stage_nb) {
  pdl_begin();
  constexpr int LPR = D / 8;          // threads per token row, 8 channels each
  constexpr int RPC = THREADS / LPR;  // rows per pass
  constexpr int NPASS = BLK / RPC;
  __shared__ float kpart[G][BLK][LPR + 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.y;
  const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
  const size_t u = (size_t)unit0 + unit;
  const size_t hrow0 = (size_t)b * sh.Hq + (size_t)g * G;
  int nb, r_unused;
  row_blocks(sh, b, nb, r_unused);
  const int j0 = blockIdx.x * sh.chunk_blocks;
  const int j1 = min(nb, j0 + sh.chunk_blocks);
  if (j0 >= j1) return;  // past the end of a shorter row

  bool headmask[G];
  bool any = MODE == 0;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    headmask[h] = MODE == 0 || sc.dense[hrow0 + h] != 0;
    any |= headmask[h];
  }
  if (!any) return;

  // the chunk's blocks to process, found by a uniform scan of the flags
  const uint8_t* bf = sc.bflags + (size_t)unit * sh.nbm;
  auto next_block = [&](int from) {
    for (int j = from; j < j1; ++j) {
      const bool key = (bf[j] & BF_KEY) != 0;
      if (MODE == 0 ? key : !key) return j;
    }
    return j1;
  };
  const int row = tid / LPR, cl = tid - row * LPR;
  // keys of block j: the staged device copy when it holds the block, else Tier 2
  const __half* kunit = t.k2 + u * st.tier2;
  const __half* sunit = kstage ? kstage + (size_t)unit * st.tier2 : nullptr;
  auto kblock = [&](int jb) { return (jb < stage_nb ? sunit : kunit) + (size_t)jb * BLK * D; };
  uint4 cur[NPASS], nxt[NPASS];
  // Certified mode promotes nearly every block, so the first block's keys are
  // requested before its flag is known (the flag and the keys then arrive
  // together); they are reloaded in the rare case that block is not promoted.
  if (MODE == 0) {
    const __half* kb = kblock(j0);
#pragma unroll
    for (int p = 0; p < NPASS; ++p)
      cur[p] = *reinterpret_cast<const uint4*>(kb + (size_t)(p * RPC + row) * D + cl * 8);
  }
  int j = next_block(j0);
  if (j >= j1) return;
  float2 qr[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 qv = *reinterpret_cast<const uint4*>(q + (hrow0 + h) * D + cl * 8);
    const __half2* qh = reinterpret_cast<const __half2*>(&qv);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(qh[k]);
      qr[h][k] = make_float2(f.x * sh.sigma, f.y * sh.sigma);
    }
  }

  if (MODE != 0 || j != j0) {
    const __half* kb = kblock(j);
#pragma unroll
    for (int p = 0; p < NPASS; ++p)
      cur[p] = *reinterpret_cast<const uint4*>(kb + (size_t)(p * RPC + row) * D + cl * 8);
  }
  while (j < j1) {
    const int jn = next_block(j + 1);
    if (jn < j1) {
      const __half* kb = kblock(jn);
#pragma unroll
      for (int p = 0; p < NPASS; ++p)
        nxt[p] = *reinterpret_cast<const uint4*>(kb + (size_t)(p * RPC + row) * D + cl * 8);
    }
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
      const __half2* kh = reinterpret_cast<const __half2*>(&cur[p]);
      float2 kf[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) kf[k] = __half22float2(kh[k]);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k) a = __ffma2_rn(qr[h][k], kf[k], a);
        kpart[h][p * RPC + row][cl] = a.x + a.y;
      }
    }
    __syncthreads();
    // warp h: the 64 logits of head h -> scratch, and the block log-mass
    for (int h = warp; h < G; h += THREADS / 32) {
      if (!headmask[h]) continue;
      float x[2];
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const int tt = lane + 32 * s2;
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < LPR; ++k) acc += kpart[h][tt][k];
        x[s2] = acc;
      }
      float* lo = sc.logits + (hrow0 + h) * sc.ls + (size_t)j * BLK;
      lo[lane] = x[0];
      lo[lane + 32] = x[1];
      if (MODE == 0) {
        const float m = warp_max(fmaxf(x[0], x[1]));
        const float ssum = warp_sum(expf(x[0] - m) + expf(x[1] - m));
        if (lane == 0) sc.ell16[(hrow0 + h) * sh.nbm + j] = m + logf(ssum);
      }
    }
    __syncthreads();
#pragma unroll
    for (int p = 0; p < NPASS; ++p) cur[p] = nxt[p];
    j = jn;
  }
}

template <int D, int G>
cudaError_t launch_promote_t(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                             const __half* q, const Scratch& sc, int mode, const __half* kstage,
                             int stage_nb, cudaStream_t s) {
  dim3 grid(sh.nchunks, sh.B * sh.Hkv);
  if (!kstage) stage_nb = 0;
  if (mode == 0)
    return launch_pdl(promote_kernel<D, G, 0>, grid, dim3(THREADS), 0, s, t, st, unit0, sh, q, sc,
                      kstage, stage_nb);
  else
    return launch_pdl(promote_kernel<D, G, 1>, grid, dim3(THREADS), 0, s, t, st, unit0, sh, q, sc,
                      kstage, stage_nb);
}

}  // namespace

cudaError_t launch_promote(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                           const __half* q, const Scratch& sc, int mode, const __half* kstage,
                           int stage_nb, cudaStream_t s) {
  if (sh.nb_max == 0) return cudaSuccess;
#define CQA_PROMOTE_CASE(DD, GG) \
  return launch_promote_t<DD, GG>(t, st, unit0, sh, q, sc, mode, kstage, stage_nb, s)
  if (sh.d == 128) {
    switch (sh.G) {
      case 1: CQA_PROMOTE_CASE(128, 1);
      case 2: CQA_PROMOTE_CASE(128, 2);
      case 4: CQA_PROMOTE_CASE(128, 4);
      case 8: CQA_PROMOTE_CASE(128, 8);
    }
  } else {
    switch (sh.G) {
      case 1: CQA_PROMOTE_CASE(64, 1);
      case 2: CQA_PROMOTE_CASE(64, 2);
      case 4: CQA_PROMOTE_CASE(64, 4);
    }
  }
#undef CQA_PROMOTE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace cqa
