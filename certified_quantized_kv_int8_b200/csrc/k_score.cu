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
// The pass streams 136 bytes per token and kv head (128 B of codes, 8 B of
// scales amortised) from HBM and writes 16 B of logits; it is bound by HBM
// bandwidth and, close behind, by fp32 issue rate, so codes are widened with
// a byte-permute into the mantissa of 2^23 and the dot products use packed
// float2 FMAs.
#include "bulk_pipe.cuh"
#include "cqa_internal.cuh"

namespace cqa {

namespace {

constexpr int WARPS = 4;

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

// v[i] holds N partial sums on each of the N lanes of an aligned lane group;
// afterwards lane l of the group holds the full sum of value index (l % N).
template <int N>
__device__ __forceinline__ float reduce_scatter(float (&v)[N], int lane) {
#pragma unroll
  for (int m = N / 2; m >= 1; m >>= 1) {
    const bool hi = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < m; ++i) {
      const float send = hi ? v[i] : v[i + m];
      const float keep = hi ? v[i + m] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  return v[0];
}

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

// Warp-level pipeline: each warp streams its (unit, block) items through
// NSTAGE shared-memory stages filled by bulk copies (codes + scales of one
// block per stage), so several blocks are in flight per warp without holding
// them in registers.  Item k of warp gw is the sealed item gw + k * nw; warps
// gw < units first compute the residual block of unit gw while their first
// copies land.
constexpr int NSTAGE = 2;

template <int D>
__host__ __device__ constexpr int stage_bytes() { return BLK * D + 4 * D; }

template <int D, int G>
__global__ void __launch_bounds__(WARPS * 32, 3)
    score_kernel(Tier1 t, Strides st, int unit0, DecodeShape sh, const __half* __restrict__ q,
                 Scratch sc, int n_sealed, int n_res) {
  constexpr int CPT = D / 16;    // lanes per token row (16 channels each)
  constexpr int RPW = 32 / CPT;  // rows covered by one warp-wide 16-byte load
  constexpr int NL = BLK / RPW;  // loads per lane per block
  constexpr int R = CPT / G;     // rows per reduce-scatter round
  constexpr int SB = stage_bytes<D>();
  static_assert(R >= 1 && NL % R == 0, "unsupported head_dim / group size");

  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ __align__(16) float lg[WARPS][G][BLK];
  __shared__ __align__(8) uint64_t bars[WARPS][NSTAGE];

  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int cc = lane % CPT, tr = lane / CPT;
  const int nw = gridDim.x * WARPS;
  const int gw = blockIdx.x * WARPS + wib;
  unsigned char* wstage = dsm + (size_t)wib * NSTAGE * SB;

  if (lane == 0) {
    for (int s2 = 0; s2 < NSTAGE; ++s2) mbar_init(&bars[wib][s2], 1);
    mbar_init_fence();
  }
  __syncwarp();

  auto issue = [&](int k) {  // lane 0: start the copies of this warp's k-th item
    const int it = gw + k * nw;
    if (it >= n_sealed) return;
    const int unit = it / sh.nb, j = it - unit * sh.nb;
    const size_t u = (size_t)unit0 + unit;
    uint64_t* bar = &bars[wib][k % NSTAGE];
    unsigned char* dst = wstage + (size_t)(k % NSTAGE) * SB;
    mbar_arrive_expect_tx(bar, SB);
    bulk_g2s(dst, t.kcodes + u * st.kcodes + (size_t)j * BLK * D, BLK * D, bar);
    bulk_g2s(dst + BLK * D, t.kscale + u * st.kscale + (size_t)j * D, 4 * D, bar);
  };
  if (lane == 0)
    for (int k = 0; k < NSTAGE; ++k) issue(k);

  if (gw < n_res) {
    const int it = n_sealed + gw;
    // residual block: exact logits from the FP16 keys kept in device memory;
      // LPR lanes per token row, 8 channels each
      constexpr int LPR = D / 8;
      constexpr int RW = 32 / LPR;  // rows per warp pass
      const int unit = it - n_sealed;
      const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
      const size_t u = (size_t)unit0 + unit;
      const int cl = lane % LPR, rl = lane / LPR;
      const __half* kr = t.kres + u * st.res;
      float2 qf[G][4];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const uint4 qv = __ldg(reinterpret_cast<const uint4*>(
            q + ((size_t)b * sh.Hq + (size_t)g * G + h) * D + cl * 8));
        const __half2* qh = reinterpret_cast<const __half2*>(&qv);
#pragma unroll
        for (int k = 0; k < 4; ++k) qf[h][k] = __half22float2(qh[k]);
      }
      for (int r0 = 0; r0 < sh.r; r0 += RW) {
        const int tok = r0 + rl;
        float2 kf[4];
        if (tok < sh.r) {
          const uint4 kv = *reinterpret_cast<const uint4*>(kr + (size_t)tok * D + cl * 8);
          const __half2* kh = reinterpret_cast<const __half2*>(&kv);
#pragma unroll
          for (int k = 0; k < 4; ++k) kf[k] = __half22float2(kh[k]);
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) kf[k] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float2 a = make_float2(0.f, 0.f);
#pragma unroll
          for (int k = 0; k < 4; ++k) a = __ffma2_rn(qf[h][k], kf[k], a);
          float v = a.x + a.y;
#pragma unroll
          for (int m = LPR / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
          if (cl == 0 && tok < sh.r) lg[wib][h][tok] = v * sh.sigma;
        }
      }
      __syncwarp();
#pragma unroll 1
      for (int h = 0; h < G; ++h) {
        const float x0 = lane < sh.r ? lg[wib][h][lane] : -INFINITY;
        const float x1 = lane + 32 < sh.r ? lg[wib][h][lane + 32] : -INFINITY;
        float* lo = sc.logits + ((size_t)b * sh.Hq + (size_t)g * G + h) * sc.ls + (size_t)sh.nb * BLK;
        if (lane < sh.r) lo[lane] = x0;
        if (lane + 32 < sh.r) lo[lane + 32] = x1;
        float lse = -INFINITY;
        if (sh.r > 0) {
          const float m = warp_max(fmaxf(x0, x1));
          const float ssum = warp_sum((x0 > -INFINITY ? expf(x0 - m) : 0.f) +
                                      (x1 > -INFINITY ? expf(x1 - m) : 0.f));
          lse = m + logf(ssum);
        }
        if (lane == 0) sc.ell_res[(size_t)b * sh.Hq + (size_t)g * G + h] = lse;
      }
      __syncwarp();
  }

  int k = 0;
  bool ok = true;
  for (; gw + k * nw < n_sealed; ++k) {
    const int it = gw + k * nw;
    const int stg = k % NSTAGE;
    ok = mbar_wait(&bars[wib][stg], (uint32_t)((k / NSTAGE) & 1), sc.err);
    if (!ok) break;
    const uint4* stage_codes = reinterpret_cast<const uint4*>(wstage + (size_t)stg * SB);
    const float* stage_scales = reinterpret_cast<const float*>(wstage + (size_t)stg * SB + BLK * D);
    {
      const int unit = it / sh.nb, j = it - unit * sh.nb;
      const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
      float s[16];
      {
        const float4* sp = reinterpret_cast<const float4*>(stage_scales + cc * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 x = sp[i];
          s[4 * i] = x.x;
          s[4 * i + 1] = x.y;
          s[4 * i + 2] = x.z;
          s[4 * i + 3] = x.w;
        }
      }
      float2 qs[G][8];
      float dp[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const uint4* qp = reinterpret_cast<const uint4*>(
            q + ((size_t)b * sh.Hq + (size_t)g * G + h) * D + cc * 16);
        uint4 qa = __ldg(qp), qb = __ldg(qp + 1);
        const __half2* qh0 = reinterpret_cast<const __half2*>(&qa);
        const __half2* qh1 = reinterpret_cast<const __half2*>(&qb);
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 qf = __half22float2(k < 4 ? qh0[k] : qh1[k - 4]);
          acc = fmaf(fabsf(qf.x), s[2 * k], acc);
          acc = fmaf(fabsf(qf.y), s[2 * k + 1], acc);
          qs[h][k] = make_float2(qf.x * s[2 * k] * sh.sigma, qf.y * s[2 * k + 1] * sh.sigma);
        }
        dp[h] = acc;
      }

#pragma unroll
      for (int i0 = 0; i0 < NL; i0 += R) {
        float v[CPT];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint4 ww = stage_codes[(i0 + r) * 32 + lane];
          float2 x[8];
          s8x4_to_f2(ww.x, x[0], x[1]);
          s8x4_to_f2(ww.y, x[2], x[3]);
          s8x4_to_f2(ww.z, x[4], x[5]);
          s8x4_to_f2(ww.w, x[6], x[7]);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float2 a = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 8; ++k) a = __ffma2_rn(qs[h][k], x[k], a);
            v[r * G + h] = a.x + a.y;
          }
        }
        const float full = reduce_scatter<CPT>(v, lane);
        const int rr = cc / G, hh = cc - rr * G;
        lg[wib][hh][RPW * (i0 + rr) + tr] = full;
      }
      // Delta: reduce the per-lane channel partials over the row's lanes
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int m = CPT / 2; m >= 1; m >>= 1) dp[h] += __shfl_xor_sync(0xffffffffu, dp[h], m);
      }
      __syncwarp();
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float x0 = lg[wib][h][lane], x1 = lg[wib][h][lane + 32];
        const float m = warp_max(fmaxf(x0, x1));
        const float ssum = warp_sum(expf(x0 - m) + expf(x1 - m));
        if (lane == 0) {
          const size_t row = ((size_t)b * sh.Hq + (size_t)g * G + h) * sh.nbm + j;
          sc.ell8[row] = m + logf(ssum);
          sc.delta[row] = 0.5f * sh.sigma * dp[h];
        }
      }
      float* lo = sc.logits + ((size_t)b * sh.Hq + (size_t)g * G) * sc.ls + (size_t)j * BLK;
      for (int e = lane; e < G * (BLK / 4); e += 32) {
        const int h = e / (BLK / 4), k = e - h * (BLK / 4);
        *reinterpret_cast<float4*>(lo + h * sc.ls + 4 * k) =
            *reinterpret_cast<const float4*>(&lg[wib][h][4 * k]);
      }
      __syncwarp();
    }
    __syncwarp();
    if (lane == 0) {
      fence_proxy_async_smem();
      issue(k + NSTAGE);
    }
  }
  if (!ok) {
    // a copy did not land in time: wait (bounded) for the ones still in flight
    for (int k2 = k + 1; k2 < k + NSTAGE && gw + k2 * nw < n_sealed; ++k2)
      mbar_wait(&bars[wib][k2 % NSTAGE], (uint32_t)((k2 / NSTAGE) & 1), nullptr);
  }
}

template <int D, int G>
cudaError_t launch_score_t(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                           const __half* q, const Scratch& sc, cudaStream_t s) {
  const int units = sh.B * sh.Hkv;
  const int n_sealed = units * sh.nb;
  // enough warps for every residual item, at most three resident CTAs per SM
  int grid = (n_sealed + 2 * WARPS - 1) / (2 * WARPS);
  const int cap = 148 * 3;
  if (grid > cap) grid = cap;
  const int need_res = (units + WARPS - 1) / WARPS;
  if (grid < need_res) grid = need_res;
  if (grid < 1) grid = 1;
  const int smem = WARPS * NSTAGE * stage_bytes<D>();
  cudaError_t e = ensure_dynamic_smem((const void*)score_kernel<D, G>, (int)smem);
  if (e != cudaSuccess) return e;
  score_kernel<D, G><<<grid, WARPS * 32, smem, s>>>(t, st, unit0, sh, q, sc, n_sealed, units);
  return cudaGetLastError();
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
