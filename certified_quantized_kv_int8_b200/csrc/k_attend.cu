// Split-K decode attention over the tiered cache with the fused value-bound
// accumulation (the softmax and P.V pass of a certified decode step), and the
// exact dense attention from Tier 2 used by the E_val post-check and by
// cqa_dense_reference.
//
// Runtime-Certified Bounded-Error Quantized Attention, Methodology §1
// (Tier 2 FP16 originals in pinned host memory, paged in on promotion and for
// the deterministic dense fallback), §2 (E_val: attention mass times eta_b
// over the blocks whose values stay INT4) and §3 (promoted blocks use FP16
// keys, tail blocks keep their INT8 scores; the FP16 block log-masses of the
// promoted blocks feed the rank-consistency check).
//
// In a certified step the logits are already final when this pass runs: the
// scoring pass wrote INT8 logits, the promotion pass replaced those of the
// promoted blocks (and, for heads that fall back to dense attention, of every
// block) with exact ones.  This pass reads them, chooses each block's values
// per head (FP16 straight from the pinned, device-mapped Tier 2 for
// value-promoted blocks and dense heads, INT4 from Tier 1 otherwise) and
// accumulates the attention mass of INT4-valued blocks times eta_b.
//
// One CTA = (kv head unit, chunk of consecutive blocks), all G query heads;
// chunk 0 also takes the exact residual block.  Per head the CTA keeps an
// online-softmax state (m, l, eta mass, o[d]) and writes it as a partial for
// the combine step.  INT4 values are folded per group:
//   sum_t p_t (s_t code_tc + z_t) = sum_t (p_t s_t) code_tc + sum_t p_t z_t.
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

// 8 INT4 codes (channels 2i in the low nibble of byte i, 2i+1 in the high one)
// -> 4 float2 (even, odd channel), exactly.
__device__ __forceinline__ void u4x8_to_f2(uint32_t w, float2 (&c)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const float2 off = make_float2(-8388608.0f, -8388608.0f);
  c[0] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650)),
                                __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650))), off);
  c[1] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7651)),
                                __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7651))), off);
  c[2] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7652)),
                                __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7652))), off);
  c[3] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7653)),
                                __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7653))), off);
}

template <int D, int G>
struct AttendSmem {
  static constexpr int LPR = D / 8;
  float lg[G][BLK];
  float pp[G][BLK];
  union {
    float kpart[G][BLK][LPR + 1];
    float red[THREADS / LPR][D];
  } u;
  float m[G], l[G], e[G], alpha[G];
};

// MODE 0: certified.  Logits come from scratch: INT8 for tail blocks, exact
//         for promoted blocks, the residual, and every block of a dense head.
//         Values per (block, head): FP16 from Tier 2 for value-promoted blocks
//         and dense heads, INT4 from Tier 1 otherwise.
// MODE 1: exact attention from Tier 2 keys and values for units holding a head
//         flagged DENSE_LATE (the E_val post-check).
// MODE 2: exact attention from Tier 2 for every head (cqa_dense_reference).
template <int D, int G, int MODE>
__global__ void __launch_bounds__(THREADS) attend_kernel(Tier1 t, Strides st, int unit0,
                                                         DecodeShape sh,
                                                         const __half* __restrict__ q,
                                                         Scratch sc) {
  pdl_begin();
  constexpr int LPR = D / 8;              // threads per token row, 8 channels each
  constexpr int RPC = THREADS / LPR;      // rows handled per pass
  constexpr int NPASS = BLK / RPC;        // passes per block
  constexpr int NG = D / VG;
  __shared__ AttendSmem<D, G> S;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.y;
  const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
  const size_t u = (size_t)unit0 + unit;
  const size_t hrow0 = (size_t)b * sh.Hq + (size_t)g * G;
  const int chunk = blockIdx.x;
  int nb, rr;
  row_blocks(sh, b, nb, rr);
  const int j0 = chunk * sh.chunk_blocks;
  const int j1 = min(nb, j0 + sh.chunk_blocks);  // j0 >= j1 past the end of a shorter row

  // per head: exact (dense) or certified mixed attention
  bool dh[G];
  bool any_dense = false, any_mixed = false;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint8_t dv = sc.dense[hrow0 + h];
    dh[h] = MODE == 0 ? (dv != 0) : true;
    any_dense |= dh[h];
    any_mixed |= !dh[h];
  }
  if (MODE == 1) {
    bool late = false;
#pragma unroll
    for (int h = 0; h < G; ++h) late |= (sc.dense[hrow0 + h] & DENSE_LATE) != 0;
    if (!late) return;
  }

  const int row = tid / LPR, cl = tid - row * LPR;  // row in pass, channel slice cl*8..cl*8+7
  float2 qr[G][4];
  if (MODE != 0) {
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
  }
  float2 acc[G][4];
  float zacc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    zacc[h] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[h][k] = make_float2(0.f, 0.f);
  }
  if (tid < G) {
    S.m[tid] = -INFINITY;
    S.l[tid] = 0.f;
    S.e[tid] = 0.f;
  }

  const uint8_t* bf = sc.bflags + ((size_t)b * sh.Hkv + g) * sh.nbm;
  const float* etap = t.eta + u * st.eta;
  const int jstart = (chunk == 0 && rr > 0) ? -1 : j0;  // -1 = the residual block
  // flags and eta_b of the next block are loaded one block ahead
  auto blk_flags = [&](int j) -> uint8_t {
    return (MODE == 0 && j >= 0 && j < j1) ? bf[j] : (uint8_t)(BF_KEY | BF_VAL);
  };
  auto blk_eta = [&](int j) -> float { return (MODE == 0 && j >= 0 && j < j1) ? etap[j] : 0.f; };
  uint8_t fl_next = blk_flags(jstart);
  float eta_next = blk_eta(jstart);
  for (int j = jstart; j < j1; ++j) {
    const bool resid = j < 0;
    const uint8_t fl = fl_next;
    const float eta_b = eta_next;
    fl_next = blk_flags(j + 1);
    eta_next = blk_eta(j + 1);
    const bool vprom = resid || (fl & BF_VAL);
    const int ntok = resid ? rr : BLK;
    const size_t tok0 = resid ? (size_t)nb * BLK : (size_t)j * BLK;  // token index
    const bool need_f16 = vprom || any_dense;
    const bool need_i4 = MODE == 0 && !vprom && any_mixed;

    // ---- this block's values, issued first: their latency overlaps the logits and softmax ----
    uint4 vv[NPASS];
    uint32_t wq[NPASS];
    float2 mt[NPASS];
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
      const int tt = p * RPC + row;
      vv[p] = make_uint4(0u, 0u, 0u, 0u);
      wq[p] = 0u;
      mt[p] = make_float2(0.f, 0.f);
      if (tt < ntok) {
        if (need_f16) {
          const __half* vsrc = resid ? t.vres + u * st.res + (size_t)tt * D
                                     : t.v2 + u * st.tier2 + (tok0 + tt) * D;
          vv[p] = *reinterpret_cast<const uint4*>(vsrc + cl * 8);
        }
        if (need_i4) {
          wq[p] = *reinterpret_cast<const uint32_t*>(
              t.vcodes + u * st.vcodes + ((size_t)j * BLK + tt) * (D / 2) + cl * 4);
          const size_t mi = u * st.vmeta + (((size_t)j * BLK + tt) * NG + (cl * 8) / VG) * 2;
          mt[p] = t.meta16 ? __half22float2(*reinterpret_cast<const __half2*>(t.vmeta_h + mi))
                           : *reinterpret_cast<const float2*>(t.vmeta + mi);
        }
      }
    }

    // ---- logits ----
    if (MODE == 0) {
      const float* lp = sc.logits + hrow0 * sc.ls + tok0;
      for (int e = tid; e < G * BLK; e += THREADS) {
        const int h = e / BLK, tt = e - h * BLK;
        S.lg[h][tt] = tt < ntok ? lp[h * sc.ls + tt] : -INFINITY;
      }
    } else {
      const __half* kb = resid ? t.kres + u * st.res : t.k2 + u * st.tier2 + tok0 * D;
      uint4 kv[NPASS];
#pragma unroll
      for (int p = 0; p < NPASS; ++p)
        kv[p] = *reinterpret_cast<const uint4*>(kb + (size_t)(p * RPC + row) * D + cl * 8);
#pragma unroll
      for (int p = 0; p < NPASS; ++p) {
        const __half2* kh = reinterpret_cast<const __half2*>(&kv[p]);
        float2 kf[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) kf[k] = __half22float2(kh[k]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float2 a = make_float2(0.f, 0.f);
#pragma unroll
          for (int k = 0; k < 4; ++k) a = __ffma2_rn(qr[h][k], kf[k], a);
          S.u.kpart[h][p * RPC + row][cl] = a.x + a.y;
        }
      }
      __syncthreads();
      for (int e = tid; e < G * BLK; e += THREADS) {
        const int h = e / BLK, tt = e - h * BLK;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < LPR; ++k) s += S.u.kpart[h][tt][k];
        S.lg[h][tt] = tt < ntok ? s : -INFINITY;
      }
    }
    __syncthreads();

    // ---- online softmax statistics, one warp per head ----
    if (warp < G) {
      const int h = warp;
      const float x0 = S.lg[h][lane], x1 = S.lg[h][lane + 32];
      const float mb = warp_max(fmaxf(x0, x1));
      const float e0 = expf(x0 - mb), e1 = expf(x1 - mb);
      const float sb = warp_sum(e0 + e1);
      const float mold = S.m[h];
      const float mnew = fmaxf(mold, mb);
      const float alpha = (mold == -INFINITY) ? 0.f : expf(mold - mnew);
      const float c = expf(mb - mnew);
      S.pp[h][lane] = e0 * c;
      S.pp[h][lane + 32] = e1 * c;
      if (lane == 0) {
        const float lb = sb * c;
        S.l[h] = S.l[h] * alpha + lb;
        float ea = S.e[h] * alpha;
        const bool int4_here = MODE == 0 && !vprom && !dh[h];  // dh[h]: head h is dense
        if (int4_here) ea += eta_b * lb;
        S.e[h] = ea;
        S.m[h] = mnew;
        S.alpha[h] = alpha;
      }
    }
    __syncthreads();

    // ---- P.V ----
    float al[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      al[h] = S.alpha[h];
      zacc[h] *= al[h];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[h][k].x *= al[h];
        acc[h][k].y *= al[h];
      }
    }
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
      const int tt = p * RPC + row;
      if (tt >= ntok) continue;
      float pw[G];
#pragma unroll
      for (int h = 0; h < G; ++h) pw[h] = S.pp[h][tt];
      float2 vf[4];
      if (need_f16) {
        const __half2* vh = reinterpret_cast<const __half2*>(&vv[p]);
#pragma unroll
        for (int k = 0; k < 4; ++k) vf[k] = __half22float2(vh[k]);
      }
      float2 cf[4];
      if (need_i4) u4x8_to_f2(wq[p], cf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (vprom || dh[h]) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            acc[h][k] = __ffma2_rn(make_float2(pw[h], pw[h]), vf[k], acc[h][k]);
        } else {
          const float ws = pw[h] * mt[p].x;
          zacc[h] = fmaf(pw[h], mt[p].y, zacc[h]);
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[h][k] = __ffma2_rn(make_float2(ws, ws), cf[k], acc[h][k]);
        }
      }
    }
    __syncthreads();
  }

  // ---- partial: sum the rows' accumulators, one head at a time ----
  const size_t pbase = ((size_t)unit * sc.max_chunks + chunk) * G;
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      S.u.red[row][cl * 8 + 2 * k] = acc[h][k].x + zacc[h];
      S.u.red[row][cl * 8 + 2 * k + 1] = acc[h][k].y + zacc[h];
    }
    __syncthreads();
    for (int c = tid; c < D; c += THREADS) {
      float s = 0.f;
      for (int r = 0; r < RPC; ++r) s += S.u.red[r][c];
      sc.part_o[(pbase + h) * D + c] = s;
    }
    __syncthreads();
  }
  if (tid < G) {
    sc.part_s[(pbase + tid) * 3 + 0] = S.m[tid];
    sc.part_s[(pbase + tid) * 3 + 1] = S.l[tid];
    sc.part_s[(pbase + tid) * 3 + 2] = S.e[tid];
  }
}

template <int D, int G>
cudaError_t launch_attend_t(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                            const __half* q, const Scratch& sc, int mode, cudaStream_t s) {
  dim3 grid(sh.nchunks, sh.B * sh.Hkv);
  if (mode == 0)
    return launch_pdl(attend_kernel<D, G, 0>, grid, dim3(THREADS), 0, s, t, st, unit0, sh, q, sc);
  else if (mode == 1)
    return launch_pdl(attend_kernel<D, G, 1>, grid, dim3(THREADS), 0, s, t, st, unit0, sh, q, sc);
  else
    return launch_pdl(attend_kernel<D, G, 2>, grid, dim3(THREADS), 0, s, t, st, unit0, sh, q, sc);
}

}  // namespace

cudaError_t launch_attend(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                          const __half* q, const Scratch& sc, int mode, cudaStream_t s) {
  if (sh.d == 128) {
    switch (sh.G) {
      case 1: return launch_attend_t<128, 1>(t, st, unit0, sh, q, sc, mode, s);
      case 2: return launch_attend_t<128, 2>(t, st, unit0, sh, q, sc, mode, s);
      case 4: return launch_attend_t<128, 4>(t, st, unit0, sh, q, sc, mode, s);
      case 8: return launch_attend_t<128, 8>(t, st, unit0, sh, q, sc, mode, s);
    }
  } else {
    switch (sh.G) {
      case 1: return launch_attend_t<64, 1>(t, st, unit0, sh, q, sc, mode, s);
      case 2: return launch_attend_t<64, 2>(t, st, unit0, sh, q, sc, mode, s);
      case 4: return launch_attend_t<64, 4>(t, st, unit0, sh, q, sc, mode, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace cqa
