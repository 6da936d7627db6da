// INT8 scoring pass: per (batch row, kv head, sealed block) the logits of the
// G query heads that share the kv head, the block log-mass ell8_b and the
// per-token score perturbation bound Delta_b; plus the exact logits of the
// residual block.
//
// Runtime-Certified Bounded-Error Quantized Attention, Methodology §3
// (adaptive top-K: a light scoring pass over the INT8 keys estimates the
// per-block attention masses) and §2 (Delta, the per-token score
// perturbation that drives E_key, from quantisation scales and the query).
//
//   logit_t = sigma * sum_c q_c * s_c * code_tc         sigma = 1/sqrt(d)
//   ell8_b  = log sum_{t in b} exp(logit_t)
//   Delta_b = sigma/2 * sum_c |q_c| * s_c               (|k - s*code| <= s/2)
//
// The pass reads 136 bytes per token and kv head (128 B of codes, 8 B of
// scales amortised) and writes 16 B of logits.  Its cost is instruction issue
// rather than HBM, so it is laid out like the certification-off pass:
//   * one CTA streams consecutive blocks of one (batch row, kv head) through
//     a ring of NST stages filled by bulk copies (codes + scales of a block);
//   * one CTA barrier per block publishes the block's scaled queries
//     (q * sigma * s_c, double-buffered by block parity) and releases the
//     previous block's stage;
//   * each warp scores 16 tokens of every block: sixteen lanes per token,
//     8 channels each, packed float2 FMAs, the G partial dots reduced with a
//     reduce-scatter whose register order is permuted per lane;
//   * each warp reduces its tokens' log-sum-exp per head; the four slices
//     merge into ell8_b after the next barrier;
//   * logits leave through shared memory as 16-byte stores.
// The residual block is scored exactly from its FP16 keys, after its blocks,
// by the CTA that holds it among its work items (it counts as two).
#include "bulk_pipe.cuh"
#include "cqa_internal.cuh"

namespace cqa {

namespace {

constexpr int NT = 128;  // threads per CTA: four warps
constexpr int NW = NT / 32;
constexpr int NST = 4;         // stages per CTA
constexpr int TPW = BLK / NW;  // tokens of each block scored by one warp
constexpr int CH = 8;          // channels per lane
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr int SCORE_CTAS_PER_SM = 5;  // grid target: resident CTAs per SM

template <int D, bool MH>
struct ScoreLayout {
  static constexpr int KB = BLK * D;          // INT8 key codes
  static constexpr int SB = (MH ? 2 : 4) * D;  // key scales (binary16 or float32)
  static constexpr int STAGE = KB + SB;
};

// four key scales of the stage as floats
template <bool MH>
__device__ __forceinline__ float4 load_scales4(const unsigned char* sbase, int c) {
  if constexpr (MH) {
    const uint2 v = *reinterpret_cast<const uint2*>(sbase + 2 * c);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
    return make_float4(a.x, a.y, b.x, b.y);
  } else {
    return *reinterpret_cast<const float4*>(sbase + 4 * c);
  }
}

__device__ __forceinline__ float swarp_max(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ float swarp_sum(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// Four signed int8 codes -> two float2, exactly: bias to unsigned, drop each
// byte into the low mantissa bits of 2^23, subtract 2^23 + 128.
__device__ __forceinline__ void s8x4_to_f2(uint32_t w, float2& a, float2& b) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 off = make_float2(-8388736.0f, -8388736.0f);
  a = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)),
                             __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651))),
                 off);
  b = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)),
                             __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653))),
                 off);
}

// 2^x by the hardware approximation (relative error about 2^-22)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int G>
struct ScoreSmem {
  float qf[G][D];                   // q * sigma
  float qs[2][G][D / CH][CH + 4];   // qf * key scale of the block, by block parity; rows padded
                                    // by 4 floats so eight lanes' 16-byte reads hit distinct banks
  float lgs[NW][G][TPW];            // each warp's logits of the current block
  float ellp[2][NW][G][2];          // each warp's (max, sum of 2^((x - max) log2 e)) per head
  uint64_t bar[NST];
};

template <int D, int G, bool MH>
__global__ void __launch_bounds__(NT, 5)
    score_kernel(Tier1 t, Strides st, int unit0, DecodeShape sh, const __half* __restrict__ q,
                 Scratch sc) {
  pdl_begin();
  using LY = ScoreLayout<D, MH>;
  constexpr int CPT = D / CH;     // lanes per token row
  constexpr int RPW = 32 / CPT;   // rows per warp instruction
  constexpr int NLI = TPW / RPW;  // logit iterations per block
  constexpr int NDUP = CPT > G ? CPT / G : 1;
  constexpr int QI = G * D / 4;   // float4 items of the scaled queries
  constexpr int NQI = (QI + NT - 1) / NT;
  static_assert(NLI >= 1 && RPW * NLI == TPW, "layout");

  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ __align__(16) ScoreSmem<D, G> S;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.y;
  const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
  const size_t u = (size_t)unit0 + unit;
  const size_t hrow0 = (size_t)b * sh.Hq + (size_t)g * G;
  const int chunk = blockIdx.x;

  for (int e = tid; e < G * D; e += NT) {
    const int h = e / D, c = e - h * D;
    S.qf[h][c] = __half2float(q[(hrow0 + h) * D + c]) * sh.sigma;
  }

  // work items of the row: its nb sealed blocks, then the residual block
  // (items nb and nb + 1 when it holds tokens); the nch CTAs of a unit take
  // floor or ceil of items / nch consecutive items
  int nb, rr;
  row_blocks(sh, b, nb, rr);
  const int items = row_items(nb, rr);
  // this unit's CTAs: its share of the grid target in proportion to its items
  const int nch =
      min((int)gridDim.x, unit_ctas(sh.sms * SCORE_CTAS_PER_SM, items, sh.items_sum, items));
  if (chunk >= nch) return;  // a unit of a shorter row has fewer CTAs than the grid's width
  const int base = items / nch, rem = items - base * nch;
  const int i0 = chunk * base + min(chunk, rem);
  const int i1 = i0 + base + (chunk < rem ? 1 : 0);
  const int j0 = i0;
  const int nblk = max(0, min(i1, nb) - i0);
  const bool do_res = i0 <= nb && nb < i1;  // the CTA holding item nb
  if (tid == 0) {
    for (int s2 = 0; s2 < NST; ++s2) mbar_init(&S.bar[s2], 1);
    mbar_init_fence();
  }
  __syncthreads();

  auto issue = [&](int k) {  // thread 0: copies of the chunk's k-th block
    if (k >= nblk) return;
    const int j = j0 + k;
    unsigned char* dst = dsm + (size_t)(k % NST) * LY::STAGE;
    uint64_t* bar = &S.bar[k % NST];
    mbar_arrive_expect_tx(bar, LY::STAGE);
    bulk_g2s(dst, t.kcodes + u * st.kcodes + (size_t)j * LY::KB, LY::KB, bar);
    const void* ksrc = MH ? (const void*)(t.kscale_h + u * st.kscale + (size_t)j * D)
                          : (const void*)(t.kscale + u * st.kscale + (size_t)j * D);
    bulk_g2s(dst + LY::KB, ksrc, LY::SB, bar);
  };
  if (tid == 0)
    for (int k = 0; k < NST; ++k) issue(k);

  // ell8 of block j from the four warps' slices
  auto finish_ell = [&](int pbuf, int j) {
    if (tid < G) {
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) mm = fmaxf(mm, S.ellp[pbuf][w][tid][0]);
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w)
        ss += S.ellp[pbuf][w][tid][1] * ex2((S.ellp[pbuf][w][tid][0] - mm) * LOG2E);
      sc.ell8[(hrow0 + tid) * sh.nbm + j] = mm + log2f(ss) * LN2;
    }
  };

  const int cc = lane % CPT, tr = lane / CPT;  // channel slice, row
  int pi = 0;                                  // head permutation of the reduce-scatter
#pragma unroll
  for (int m = CPT / 2, n = G; m >= 1; m >>= 1, n >>= 1)
    if (n > 1 && (cc & m)) pi |= n / 2;
  const bool owner = tr == 0 && (cc & (NDUP - 1)) == 0;  // one lane per head of the warp

  bool ok = true;
  int k = 0;
  for (; k < nblk; ++k) {
    const int j = j0 + k;
    const int stg = k % NST;
    const bool got = mbar_wait(&S.bar[stg], (uint32_t)((k / NST) & 1), sc.err);
    const unsigned char* sp = dsm + (size_t)stg * LY::STAGE;
    const unsigned char* ks = sp + LY::KB;

    // scaled queries of this block and Delta_b = sum |qs| / 2
#pragma unroll
    for (int i = 0; i < NQI; ++i) {
      const int e = tid + i * NT;
      if (e - lane < QI) {  // warp-uniform
        const bool act = e < QI;
        const int h = act ? e / (D / 4) : 0, c = act ? 4 * (e % (D / 4)) : 0;
        const float4 kq = load_scales4<MH>(ks, c);
        const float4 qv = *reinterpret_cast<const float4*>(&S.qf[h][c]);
        const float4 r = make_float4(qv.x * kq.x, qv.y * kq.y, qv.z * kq.z, qv.w * kq.w);
        if (act) *reinterpret_cast<float4*>(&S.qs[k & 1][h][c / CH][c % CH]) = r;
        float sa = act ? (fabsf(r.x) + fabsf(r.y)) + (fabsf(r.z) + fabsf(r.w)) : 0.f;
#pragma unroll
        for (int m = D / 8; m >= 1; m >>= 1) sa += __shfl_xor_sync(0xffffffffu, sa, m);
        if (act && c == 0) sc.delta[(hrow0 + h) * sh.nbm + j] = 0.5f * sa;
      }
    }
    if (__syncthreads_or(!got)) {
      ok = false;
      break;
    }
    if (tid == 0 && k >= 1) {
      fence_proxy_async_smem();
      issue(k - 1 + NST);  // the previous block's stage is free
    }
    if (k >= 1) finish_ell((k - 1) & 1, j - 1);

    // ---- logits of the warp's 16 tokens: lane (tr, cc) scores rows tr + RPW*li ----
    float x[NLI];
    {
      float2 qr[G][CH / 2];  // register r: head r ^ pi
#pragma unroll
      for (int r = 0; r < G; ++r) {
        const float4* qp = reinterpret_cast<const float4*>(&S.qs[k & 1][r ^ pi][cc][0]);
#pragma unroll
        for (int i = 0; i < CH / 4; ++i) {
          const float4 v = qp[i];
          qr[r][2 * i] = make_float2(v.x, v.y);
          qr[r][2 * i + 1] = make_float2(v.z, v.w);
        }
      }
#pragma unroll
      for (int li = 0; li < NLI; ++li) {
        const int row = warp * TPW + li * RPW + tr;
        const uint2 wd = *reinterpret_cast<const uint2*>(sp + (size_t)row * D + cc * CH);
        float2 k0, k1, k2, k3;
        s8x4_to_f2(wd.x, k0, k1);
        s8x4_to_f2(wd.y, k2, k3);
        float a[G];
#pragma unroll
        for (int r = 0; r < G; ++r) {
          float2 a2 = __fmul2_rn(qr[r][0], k0);
          a2 = __ffma2_rn(qr[r][1], k1, a2);
          a2 = __ffma2_rn(qr[r][2], k2, a2);
          a2 = __ffma2_rn(qr[r][3], k3, a2);
          a[r] = a2.x + a2.y;
        }
        // reduce-scatter over the CPT lanes of the row: level m halves the heads held
#pragma unroll
        for (int m = CPT / 2, n = G; m >= 1; m >>= 1) {
          if (n > 1) {
#pragma unroll
            for (int r = 0; r < G / 2; ++r)
              if (r < n / 2) a[r] += __shfl_xor_sync(0xffffffffu, a[r + n / 2], m);
            n >>= 1;
          } else {
            a[0] += __shfl_xor_sync(0xffffffffu, a[0], m);
          }
        }
        x[li] = a[0];  // head pi, row warp*TPW + li*RPW + tr
      }
    }

    // ---- the warp's slice of ell8 and its logits ----
    float mb = x[0];
#pragma unroll
    for (int li = 1; li < NLI; ++li) mb = fmaxf(mb, x[li]);
#pragma unroll
    for (int m = CPT; m < 32; m <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, m));
    const float mb2 = mb * LOG2E;
    float es = 0.f;
#pragma unroll
    for (int li = 0; li < NLI; ++li) es += ex2(fmaf(x[li], LOG2E, -mb2));
#pragma unroll
    for (int m = CPT; m < 32; m <<= 1) es += __shfl_xor_sync(0xffffffffu, es, m);
    if (owner) {
      S.ellp[k & 1][warp][pi][0] = mb;
      S.ellp[k & 1][warp][pi][1] = es;
#pragma unroll
      for (int li = 0; li < NLI; ++li) S.lgs[warp][pi][li * RPW + tr] = x[li];
    }
    if (tr > 0 && (cc & (NDUP - 1)) == 0) {
#pragma unroll
      for (int li = 0; li < NLI; ++li) S.lgs[warp][pi][li * RPW + tr] = x[li];
    }
    __syncwarp();
    if (lane < G * TPW / 4) {
      const int h = lane / (TPW / 4), t4 = lane % (TPW / 4);
      const float4 v = *reinterpret_cast<const float4*>(&S.lgs[warp][h][4 * t4]);
      *reinterpret_cast<float4*>(sc.logits + (hrow0 + h) * sc.ls + (size_t)j * BLK +
                                 warp * TPW + 4 * t4) = v;
    }
    __syncwarp();
  }
  if (__syncthreads_or(!ok)) {
    // let the copies still in flight land before the CTA exits
    if (tid == 0) {
      const int hi = min(nblk - 1, k == 0 ? NST - 1 : k + NST - 2);
      for (int k2 = k; k2 <= hi; ++k2)
        mbar_wait(&S.bar[k2 % NST], (uint32_t)((k2 / NST) & 1), nullptr);
    }
    return;
  }
  if (nblk > 0) finish_ell((nblk - 1) & 1, j0 + nblk - 1);

  // ---- the residual block (item nb), by the CTA holding that item: exact logits from
  // the FP16 keys in device memory ----
  if (do_res) {
    float* lg = reinterpret_cast<float*>(dsm);  // [G][BLK]
    const int r = rr;
    const __half* kr = t.kres + u * st.res;
    constexpr int CPL = D / 32;
    // four tokens per warp at a time: their key loads and the 4*G reductions are
    // independent, so their latencies overlap
    for (int t0 = 4 * warp; t0 < r; t0 += 4 * NW) {
      float kf[4][CPL];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int i = 0; i < CPL; i += 2) {
          float2 f = make_float2(0.f, 0.f);
          if (t0 + k < r)
            f = __half22float2(*reinterpret_cast<const __half2*>(kr + (size_t)(t0 + k) * D +
                                                                 lane * CPL + i));
          kf[k][i] = f.x;
          kf[k][i + 1] = f.y;
        }
      }
      float v[4][G];
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float a = 0.f;
#pragma unroll
          for (int i = 0; i < CPL; ++i) a = fmaf(S.qf[h][lane * CPL + i], kf[k][i], a);
          v[k][h] = a;
        }
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int h = 0; h < G; ++h) v[k][h] += __shfl_xor_sync(0xffffffffu, v[k][h], m);
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int h = 0; h < G; ++h)
            if (t0 + k < r) lg[h * BLK + t0 + k] = v[k][h];
      }
    }
    __syncthreads();
    for (int h = warp; h < G; h += NW) {
      const float x0 = lane < r ? lg[h * BLK + lane] : -INFINITY;
      const float x1 = lane + 32 < r ? lg[h * BLK + lane + 32] : -INFINITY;
      float* lo = sc.logits + (hrow0 + h) * sc.ls + (size_t)nb * BLK;
      if (lane < r) lo[lane] = x0;
      if (lane + 32 < r) lo[lane + 32] = x1;
      float lse = -INFINITY;
      if (r > 0) {
        const float m = swarp_max(fmaxf(x0, x1));
        const float ssum = swarp_sum((lane < r ? expf(x0 - m) : 0.f) +
                                     (lane + 32 < r ? expf(x1 - m) : 0.f));
        lse = m + logf(ssum);
      }
      if (lane == 0) sc.ell_res[hrow0 + h] = lse;
    }
  }
}

// Grid width: the most CTAs any unit receives.  Units share sms * 5 CTAs (five
// resident per SM hold the whole grid, one wave) in proportion to their work
// items, at most one CTA per item.
int score_chunks(const DecodeShape& sh) {
  int w = 1;
  for (int b = 0; b < sh.B; ++b) {
    const int T = sh.lens_host[b], nb = T / BLK, items = row_items(nb, T - nb * BLK);
    const int n = unit_ctas(sh.sms * SCORE_CTAS_PER_SM, items, sh.items_sum, items);
    w = n > w ? n : w;
  }
  return w;
}

template <int D, int G, bool MH>
cudaError_t launch_score_mh(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                            const __half* q, const Scratch& sc, cudaStream_t s) {
  const int nch = score_chunks(sh);
  const int smem = NST * ScoreLayout<D, MH>::STAGE;
  cudaError_t e = ensure_dynamic_smem((const void*)score_kernel<D, G, MH>, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(score_kernel<D, G, MH>, dim3(nch, sh.B * sh.Hkv), dim3(NT), smem, s, t, st,
                    unit0, sh, q, sc);
}

template <int D, int G>
cudaError_t launch_score_t(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                           const __half* q, const Scratch& sc, cudaStream_t s) {
  return t.meta16 ? launch_score_mh<D, G, true>(t, st, unit0, sh, q, sc, s)
                  : launch_score_mh<D, G, false>(t, st, unit0, sh, q, sc, s);
}

}  // namespace

cudaError_t launch_score(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                         const __half* q, const Scratch& sc, cudaStream_t s) {
  if (sh.d == 128) {
    switch (sh.G) {
      case 1: return launch_score_t<128, 1>(t, st, unit0, sh, q, sc, s);
      case 2: return launch_score_t<128, 2>(t, st, unit0, sh, q, sc, s);
      case 4: return launch_score_t<128, 4>(t, st, unit0, sh, q, sc, s);
      case 8: return launch_score_t<128, 8>(t, st, unit0, sh, q, sc, s);
    }
  } else {
    switch (sh.G) {
      case 1: return launch_score_t<64, 1>(t, st, unit0, sh, q, sc, s);
      case 2: return launch_score_t<64, 2>(t, st, unit0, sh, q, sc, s);
      case 4: return launch_score_t<64, 4>(t, st, unit0, sh, q, sc, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace cqa
