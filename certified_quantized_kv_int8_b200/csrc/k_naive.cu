// The INT8/INT4 decode path with certification off: one streaming pass over
// Tier 1 that scores the INT8 keys, runs the online softmax and accumulates
// the INT4 values into split-K partials, and a combine kernel, launched as a
// programmatic dependent of the pass, that merges them and reports the
// outputs, E_key and E_val.
//
// Runtime-Certified Bounded-Error Quantized Attention, Experimental Results
// (the naive INT8/INT4 baseline, without certification) and Methodology §2
// (the bounds still apply: with nothing promoted, every sealed block is in
// the tail, so E_key uses dT = dA = max Delta and the INT8 tail mass
// m8T = 1 - m_res, and E_val sums attention mass times eta_b over all
// sealed blocks).
//
// One CTA streams a chunk of consecutive blocks of one (batch row, kv head)
// through a ring of NST shared-memory stages filled by bulk copies (INT8
// codes, key scales, INT4 codes, value scale/offset and the 16 aligned bytes
// of eta holding eta_b, of one block per stage): 14.5 KiB per block for
// head_dim 128, every byte of Tier 1 read once.  The issuing thread never
// waits for a load of its own, so the copies leave as soon as a stage frees.
//
// The pass is bound by instruction issue and the FP32 pipe rather than by HBM
// (per token and kv head: 128 INT8 and 128 INT4 conversions and 2*G*head_dim
// multiply-adds against 232 bytes), so the layout is chosen to spend few
// instructions besides those:
//   * one CTA barrier per block: it publishes the block's scaled queries
//     (double-buffered by block parity) and releases the previous block's
//     stage to the copy engine;
//   * each warp owns 16 tokens of every block and keeps its own online
//     softmax state, so the softmax and the P.V step need only warp-level
//     synchronisation; the four warps' states merge once per chunk;
//   * logits: sixteen lanes per token, 8 channels each; the G partial dots are
//     reduced with a reduce-scatter whose register order is permuted per lane
//     (register r of a lane holds head r ^ pi(lane)), so no selects are needed
//     and each level halves the values in flight;
//   * logits are kept in base 2 (queries pre-scaled by log2 e) so every
//     exponential is one exp2;
//   * INT4 codes become floats without an FP32 operation: each nibble is
//     shifted under the exponent of 16 (even channels, value 16 + n) or of
//     256 (odd channels, value 256 + n) with one LOP3; the constant is removed
//     once per chunk with the per-group sum of weights the softmax lanes keep
//     (Sum w (C + n) - C Sum w), which leaves the FP32 pipe to the
//     multiply-adds;
//   * the value scale is folded into the attention weight per (token, group,
//     head) by the softmax lanes, which also accumulate the offset term.
#include "bulk_pipe.cuh"
#include "cqa_internal.cuh"
#include "split_merge.cuh"

namespace cqa {

namespace {

constexpr int NT = 128;  // threads per CTA: four warps
constexpr int NW = NT / 32;
constexpr int NST = 3;         // stages per CTA
constexpr int TPW = BLK / NW;  // tokens of each block handled by one warp
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr int NAIVE_CTAS_PER_SM = 4;  // grid target: resident CTAs per SM

// Most CTAs one unit with nb sealed blocks takes: one partial slot stays for
// the residual block, and each CTA gets at least 4 items (below that the
// per-CTA start-up and the merge of more partials cost more than the
// parallelism gains: 8K context, -10%).
__host__ __device__ __forceinline__ int naive_cap(int nb, int max_chunks) {
  const int c = (nb + 4) / 4;
  return c < max_chunks - 1 ? c : max_chunks - 1;
}

template <int D, bool MH>
struct NaiveLayout {
  static constexpr int MBY = MH ? 2 : 4;               // bytes of one metadata value
  static constexpr int KB = BLK * D;                   // INT8 key codes
  static constexpr int SB = MBY * D;                   // key scales
  static constexpr int VB = BLK * D / 2;               // INT4 value codes
  static constexpr int MB = BLK * (D / VG) * 2 * MBY;  // value scale/offset
  static constexpr int STAGE = KB + SB + VB + MB;
};

// four key scales, and one (scale, offset) pair, of a stage as floats
// (binary16 metadata is widened, exactly)
template <bool MH>
__device__ __forceinline__ float4 stage_scales4(const unsigned char* sbase, int c) {
  if constexpr (MH) {
    const uint2 v = *reinterpret_cast<const uint2*>(sbase + 2 * c);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
    return make_float4(a.x, a.y, b.x, b.y);
  } else {
    return *reinterpret_cast<const float4*>(sbase + 4 * c);
  }
}

template <bool MH>
__device__ __forceinline__ float2 stage_meta(const unsigned char* mbase, int i) {
  if constexpr (MH) return __half22float2(*reinterpret_cast<const __half2*>(mbase + 4 * i));
  else return *reinterpret_cast<const float2*>(mbase + 8 * i);
}

// channels per lane in the logit step.  The lane holds its channels' scaled
// queries for every head in registers; 8 channels (16 lanes per token) keep the
// kernel within 128 registers with the P.V accumulators, where 16 channels
// spill and issue fewer instructions per cycle, for the same count.
template <int G>
struct NaiveLanes {
  static constexpr int CH = 8;
};

__device__ __forceinline__ float nwarp_max(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ float nwarp_sum(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// four INT8 codes -> floats: bias to unsigned, place each byte in the
// mantissa of 2^23, subtract 2^23 + 128 (exact)
__device__ __forceinline__ void s8x4_f2(uint32_t w, float2& a, float2& b) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 off = make_float2(-8388736.0f, -8388736.0f);
  a = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)),
                             __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651))), off);
  b = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)),
                             __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653))), off);
}

// eight INT4 codes (nibble k = channel k) -> floats C_k + n_k without an FP32
// operation: even nibbles are shifted to mantissa bits 19-22 under the exponent
// of 16 (value 16 + n), odd ones to bits 15-18 under the exponent of 256
// (value 256 + n); c[p] = (channel 2p, channel 2p + 1)
__device__ __forceinline__ void u4x8_biased(uint32_t w, float2 (&c)[4]) {
  const uint32_t s0 = w << 19;  // n0 -> 19
  const uint32_t s1 = w << 11;  // n1 -> 15, n2 -> 19
  const uint32_t s2 = w << 3;   // n3 -> 15, n4 -> 19
  const uint32_t s3 = w >> 5;   // n5 -> 15, n6 -> 19
  const uint32_t s4 = w >> 13;  // n7 -> 15
  constexpr uint32_t E16 = 0x41800000u, E256 = 0x43800000u;
  constexpr uint32_t M19 = 0xFu << 19, M15 = 0xFu << 15;
  c[0] = make_float2(__uint_as_float((s0 & M19) | E16), __uint_as_float((s1 & M15) | E256));
  c[1] = make_float2(__uint_as_float((s1 & M19) | E16), __uint_as_float((s2 & M15) | E256));
  c[2] = make_float2(__uint_as_float((s2 & M19) | E16), __uint_as_float((s3 & M15) | E256));
  c[3] = make_float2(__uint_as_float((s3 & M19) | E16), __uint_as_float((s4 & M15) | E256));
}


// 2^x by the hardware approximation (relative error about 2^-22; flushes
// results below 2^-126 to zero, which only drops weights that small)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// floats of the stage area a CTA reuses after its last block: the per-warp
// states of the chunk end, then the residual block's logits and statistics
template <int D, int G>
struct NaiveScratchFloats {
  static constexpr int RES = G * BLK + 2 * G;
  static constexpr int MAIN = NW * G * (D + 2 * (D / VG) + 3);
  static constexpr int N = RES > MAIN ? RES : MAIN;
};

template <int D, int G>
struct NaiveSmem {
  static constexpr int CH = NaiveLanes<G>::CH;
  float qf[G][D];                  // q * sigma * log2(e)
  float qs[2][G][D / CH][CH + 4];  // qf * key scale of the block, by block parity; rows padded
                                   // by 4 floats so eight lanes' 16-byte reads hit distinct banks
  float ws[NW][TPW][D / VG][G];    // attention weight * value scale per (token, group, head)
  float alpha[NW][G];              // rescale factor of each warp's running state
  float ellp[2][NW][G];            // trace: log2-sum-exp of each warp's tokens of a block
  float dmax[G];
  __align__(16) float eta[NST][4];  // the 16-byte run of eta holding eta_b of each stage's block
  uint64_t bar[NST];
};

__device__ double naive_e_key(double dT, double dA, double m8T) {
  const double a = m8T * exp(dT);
  const double m_ub = a > 0.0 ? a / (a + (1.0 - m8T) * exp(-dA)) : 0.0;
  return fmin(tanh(0.5 * dT), m_ub * expm1(2.0 * dT));
}

template <int D, int G, bool MH>
__global__ void __launch_bounds__(NT, G >= 8 ? 2 : 4)
    naive_kernel(Tier1 t, Strides st, int unit0, DecodeShape sh, const __half* __restrict__ q,
                 Scratch sc, int trace,
                 float* __restrict__ out, float* __restrict__ e_key, float* __restrict__ e_val,
                 uint8_t* __restrict__ rung) {
  pdl_begin();
  using LY = NaiveLayout<D, MH>;
  constexpr int NG = D / VG;
  constexpr int CH = NaiveLanes<G>::CH;
  constexpr int CPT = D / CH;        // lanes per token row in the logit step
  constexpr int RPW = 32 / CPT;      // rows per warp instruction
  constexpr int NLI = TPW / RPW;     // logit iterations per block
  constexpr int LPT = D / 8;         // lanes per token row in the P.V step (8 channels each)
  constexpr int TPI = 32 / LPT;
  constexpr int NPI = TPW / TPI;
  constexpr int NDUP = CPT > G ? CPT / G : 1;  // lanes holding the same (token, head) logit
  constexpr int GPL = NG > NDUP ? NG / NDUP : 1;  // value groups per softmax lane
  constexpr int QI = G * D / 4;                   // float4 items of the scaled queries
  constexpr int NQI = (QI + NT - 1) / NT;
  static_assert(NLI >= 1 && NPI >= 1 && RPW * NLI == TPW, "layout");

  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ __align__(16) NaiveSmem<D, G> S;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.y;
  const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
  const size_t u = (size_t)unit0 + unit;
  const size_t hrow0 = (size_t)b * sh.Hq + (size_t)g * G;
  const int chunk = blockIdx.x;
  const size_t pbase = ((size_t)unit * sc.max_chunks + chunk) * G;
  const float s2 = sh.sigma * LOG2E;

  for (int e = tid; e < G * D; e += NT) {
    const int h = e / D, c = e - h * D;
    S.qf[h][c] = __half2float(q[(hrow0 + h) * D + c]) * s2;
  }
  if (tid < G) S.dmax[tid] = 0.f;  // published by the barrier before the first block

  // work items of the row: its nb sealed blocks, then the residual block
  // (items nb and nb + 1 when it holds tokens); the nch CTAs of a unit take
  // floor or ceil of items / nch consecutive items
  int nb, rr;
  row_blocks(sh, b, nb, rr);
  const int items = row_items(nb, rr);
  // this unit's CTAs: its share of the grid target in proportion to its items
  const int nch = min((int)gridDim.x, unit_ctas(sh.sms * NAIVE_CTAS_PER_SM, items, sh.items_sum,
                                                naive_cap(nb, sc.max_chunks)));
  if (chunk >= nch) return;  // a unit of a shorter row has fewer CTAs than the grid's width
  const int base = items / nch, rem = items - base * nch;
  const int i0 = chunk * base + min(chunk, rem);
  const int i1 = i0 + base + (chunk < rem ? 1 : 0);
  const int j0 = i0;
  const int nblk = max(0, min(i1, nb) - i0);
  const bool do_res = i0 <= nb && nb < i1;  // the CTA holding item nb
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) mbar_init(&S.bar[s], 1);
    mbar_init_fence();
  }
  __syncthreads();

  auto issue = [&](int k) {  // thread 0: copies of the chunk's k-th block
    if (k >= nblk) return;
    const int j = j0 + k;
    unsigned char* dst = dsm + (size_t)(k % NST) * LY::STAGE;
    uint64_t* bar = &S.bar[k % NST];
    const size_t ei = u * st.eta + j;  // eta_b arrives with the block: 16 aligned bytes holding it
    mbar_arrive_expect_tx(bar, LY::STAGE + 16);
    bulk_g2s(&S.eta[k % NST][0], t.eta + (ei & ~(size_t)3), 16, bar);
    bulk_g2s(dst, t.kcodes + u * st.kcodes + (size_t)j * LY::KB, LY::KB, bar);
    const size_t ko = u * st.kscale + (size_t)j * D, mo = u * st.vmeta + (size_t)j * BLK * NG * 2;
    bulk_g2s(dst + LY::KB, MH ? (const void*)(t.kscale_h + ko) : (const void*)(t.kscale + ko),
             LY::SB, bar);
    bulk_g2s(dst + LY::KB + LY::SB, t.vcodes + u * st.vcodes + (size_t)j * LY::VB, LY::VB, bar);
    bulk_g2s(dst + LY::KB + LY::SB + LY::VB,
             MH ? (const void*)(t.vmeta_h + mo) : (const void*)(t.vmeta + mo), LY::MB, bar);
  };
  // Only the first stage now: the grid's first blocks (one per CTA) then reach
  // HBM ahead of any CTA's later stages, which thread 0 issues once block 0 has
  // landed, so every CTA starts computing sooner.
  if (tid == 0) issue(0);

  // lane roles
  const int cc = lane % CPT, tr = lane / CPT;  // logit step: channel slice, row
  int pi = 0;                                  // head permutation of the reduce-scatter
#pragma unroll
  for (int m = CPT / 2, n = G; m >= 1; m >>= 1, n >>= 1)
    if (n > 1 && (cc & m)) pi |= n / 2;
  const int dup = cc & (NDUP - 1);
  const bool owner = tr == 0 && dup == 0;  // one lane per head of the warp
  const int cl = lane % LPT, ts = lane / LPT;  // P.V step: channel slice, row
  const int gq = cl * 8 / VG;

  float2 acc[G][4];  // P.V accumulators, channel 8*cl + k carries C = 16 (k even) or 256 (k odd)
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[h][i] = make_float2(0.f, 0.f);
  float zl[GPL], wl[GPL];  // offset term and weight sum, per owned group of head pi
#pragma unroll
  for (int i = 0; i < GPL; ++i) zl[i] = wl[i] = 0.f;
  float mrun = -INFINITY, lrun = 0.f, erun = 0.f;  // running state of head pi (base 2)

  bool ok = true;
  int k = 0;
  for (; k < nblk; ++k) {
    const int j = j0 + k;
    const int stg = k % NST;
    const bool got = mbar_wait(&S.bar[stg], (uint32_t)((k / NST) & 1), sc.err);
    const unsigned char* sp = dsm + (size_t)stg * LY::STAGE;
    const unsigned char* ks = sp + LY::KB;
    const uint8_t* vc = sp + LY::KB + LY::SB;
    const unsigned char* vm = sp + LY::KB + LY::SB + LY::VB;

    // scaled queries of this block and Delta_b (base 2: sum |qs| / 2)
#pragma unroll
    for (int i = 0; i < NQI; ++i) {
      const int e = tid + i * NT;
      if (e - lane < QI) {  // warp-uniform
        const bool act = e < QI;
        const int h = act ? e / (D / 4) : 0, c = act ? 4 * (e % (D / 4)) : 0;
        const float4 kq = stage_scales4<MH>(ks, c);
        const float4 qv = *reinterpret_cast<const float4*>(&S.qf[h][c]);
        const float4 r = make_float4(qv.x * kq.x, qv.y * kq.y, qv.z * kq.z, qv.w * kq.w);
        if (act) *reinterpret_cast<float4*>(&S.qs[k & 1][h][c / CH][c % CH]) = r;
        float sa = act ? (fabsf(r.x) + fabsf(r.y)) + (fabsf(r.z) + fabsf(r.w)) : 0.f;
#pragma unroll
        for (int m = D / 8; m >= 1; m >>= 1) sa += __shfl_xor_sync(0xffffffffu, sa, m);
        if (act && c == 0) {
          S.dmax[h] = fmaxf(S.dmax[h], sa);  // one thread per head
          if (trace) sc.delta[(hrow0 + h) * sh.nbm + j] = 0.5f * sa * LN2;
        }
      }
    }
    if (__syncthreads_or(!got)) {
      ok = false;
      break;
    }
    if (tid == 0 && k == 0)
      for (int k2 = 1; k2 < NST; ++k2) issue(k2);
    if (tid == 0 && k >= 1) {
      fence_proxy_async_smem();
      issue(k - 1 + NST);  // the previous block's stage is free
    }
    if (trace && k >= 1 && tid < G) {
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) mm = fmaxf(mm, S.ellp[(k - 1) & 1][w][tid]);
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) ss += exp2f(S.ellp[(k - 1) & 1][w][tid] - mm);
      sc.ell8[(hrow0 + tid) * sh.nbm + j - 1] = (mm + log2f(ss)) * LN2;
      if (tid == 0) sc.bflags[(size_t)unit * sh.nbm + j - 1] = 0;  // nothing promoted
    }

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
        const uint32_t* kw = reinterpret_cast<const uint32_t*>(sp + (size_t)row * D + cc * CH);
        uint32_t wd[CH / 4];
        if constexpr (CH == 16) {
          const uint4 v = *reinterpret_cast<const uint4*>(kw);
          wd[0] = v.x; wd[1] = v.y; wd[2] = v.z; wd[3] = v.w;
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(kw);
          wd[0] = v.x; wd[1] = v.y;
        }
        float2 a2[G];
#pragma unroll
        for (int r = 0; r < G; ++r) a2[r] = make_float2(0.f, 0.f);
#pragma unroll
        for (int wi = 0; wi < CH / 4; ++wi) {
          float2 x0, x1;
          s8x4_f2(wd[wi], x0, x1);
#pragma unroll
          for (int r = 0; r < G; ++r) {
            a2[r] = __ffma2_rn(qr[r][2 * wi], x0, a2[r]);
            a2[r] = __ffma2_rn(qr[r][2 * wi + 1], x1, a2[r]);
          }
        }
        float a[G];
#pragma unroll
        for (int r = 0; r < G; ++r) a[r] = a2[r].x + a2[r].y;
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

    // ---- online softmax of head pi over the warp's tokens ----
    float mb = x[0];
#pragma unroll
    for (int li = 1; li < NLI; ++li) mb = fmaxf(mb, x[li]);
#pragma unroll
    for (int m = CPT; m < 32; m <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, m));
    const float mnew = fmaxf(mrun, mb);
    const float alpha = ex2(mrun - mnew);  // 0 on the first block
    float p[NLI], ps = 0.f;
#pragma unroll
    for (int li = 0; li < NLI; ++li) {
      p[li] = ex2(x[li] - mnew);
      ps += p[li];
    }
#pragma unroll
    for (int m = CPT; m < 32; m <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, m);
    lrun = fmaf(lrun, alpha, ps);
    erun = fmaf(erun, alpha, S.eta[stg][(u * st.eta + j) & 3] * ps);
    mrun = mnew;
    if (trace) {
      float es = 0.f;
#pragma unroll
      for (int li = 0; li < NLI; ++li) es += ex2(x[li] - mb);
#pragma unroll
      for (int m = CPT; m < 32; m <<= 1) es += __shfl_xor_sync(0xffffffffu, es, m);
      if (owner) S.ellp[k & 1][warp][pi] = mb + log2f(es);
    }
    if (owner) S.alpha[warp][pi] = alpha;
    const bool rescale = __any_sync(0xffffffffu, alpha != 1.f);
    // value scale folded into the weights; offset term accumulated here
    if (dup * GPL < NG) {
#pragma unroll
      for (int i = 0; i < GPL; ++i) {
        zl[i] *= alpha;
        wl[i] *= alpha;
      }
#pragma unroll
      for (int li = 0; li < NLI; ++li) {
        const int tok = li * RPW + tr;
        const int mrow = (warp * TPW + tok) * NG + dup * GPL;
#pragma unroll
        for (int i = 0; i < GPL; ++i) {
          const float2 sz = stage_meta<MH>(vm, mrow + i);
          const float wv = p[li] * sz.x;
          S.ws[warp][tok][dup * GPL + i][pi] = wv;
          wl[i] += wv;
          zl[i] = fmaf(p[li], sz.y, zl[i]);
        }
      }
    }
    __syncwarp();

    // ---- P.V: lane (ts, cl) accumulates channels 8*cl .. 8*cl+7 of rows ts + TPI*i ----
    if (rescale) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float al = S.alpha[warp][h];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[h][i].x *= al;
          acc[h][i].y *= al;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NPI; ++i) {
      const int tok = i * TPI + ts;
      const uint32_t w =
          *reinterpret_cast<const uint32_t*>(vc + (size_t)(warp * TPW + tok) * (D / 2) + cl * 4);
      float wsv[G];
      if constexpr (G % 4 == 0) {
#pragma unroll
        for (int h = 0; h < G; h += 4) {
          const float4 v = *reinterpret_cast<const float4*>(&S.ws[warp][tok][gq][h]);
          wsv[h] = v.x; wsv[h + 1] = v.y; wsv[h + 2] = v.z; wsv[h + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int h = 0; h < G; ++h) wsv[h] = S.ws[warp][tok][gq][h];
      }
      float2 cf[4];
      u4x8_biased(w, cf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float2 ww = make_float2(wsv[h], wsv[h]);
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) acc[h][q2] = __ffma2_rn(ww, cf[q2], acc[h][q2]);
      }
    }
  }
  if (!ok) {
    // let the copies still in flight land before the CTA exits, and leave empty
    // partials (the status word already reports that the results are invalid)
    if (tid == 0) {
      const int hi = min(nblk - 1, k == 0 ? 0 : k + NST - 2);
      for (int k2 = k; k2 <= hi; ++k2)
        mbar_wait(&S.bar[k2 % NST], (uint32_t)((k2 / NST) & 1), nullptr);
    }
    if (tid < G) {
      for (int s2 = 0; s2 < (do_res ? 2 : 1); ++s2) {
        const size_t pb = s2 ? ((size_t)unit * sc.max_chunks + nch) * G : pbase;
        sc.part_s[(pb + tid) * 3 + 0] = -INFINITY;
        sc.part_s[(pb + tid) * 3 + 1] = 0.f;
        sc.part_s[(pb + tid) * 3 + 2] = 0.f;
        sc.part_x[(pb + tid) * 3 + 0] = 0.f;
        sc.part_x[(pb + tid) * 3 + 1] = -INFINITY;
        sc.part_x[(pb + tid) * 3 + 2] = 0.f;
      }
    }
    return;
  }
  __syncthreads();  // every warp is past its last block: the stages are free
  if (trace && nblk > 0 && tid < G) {
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mm = fmaxf(mm, S.ellp[(nblk - 1) & 1][w][tid]);
    float ss = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) ss += exp2f(S.ellp[(nblk - 1) & 1][w][tid] - mm);
    sc.ell8[(hrow0 + tid) * sh.nbm + j0 + nblk - 1] = (mm + log2f(ss)) * LN2;
    if (tid == 0) sc.bflags[(size_t)unit * sh.nbm + j0 + nblk - 1] = 0;
  }

  // ---- merge the four warps' states ----
  float* ow = reinterpret_cast<float*>(dsm);  // [NW][G][D] unscaled P.V of each warp
  float* zw = ow + NW * G * D;                // [NW][G][NG][2] offset term minus C * weight sum
  float* mw = zw + NW * G * NG * 2;           // [NW][G][3] m, l, e
#pragma unroll
  for (int m = LPT; m < 32; m <<= 1)
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[h][i].x += __shfl_xor_sync(0xffffffffu, acc[h][i].x, m);
        acc[h][i].y += __shfl_xor_sync(0xffffffffu, acc[h][i].y, m);
      }
  if (ts == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<float2*>(&ow[(warp * G + h) * D + cl * 8 + 2 * i]) =
            acc[h][i];
  }
#pragma unroll
  for (int m = CPT; m < 32; m <<= 1)
#pragma unroll
    for (int i = 0; i < GPL; ++i) {
      zl[i] += __shfl_xor_sync(0xffffffffu, zl[i], m);
      wl[i] += __shfl_xor_sync(0xffffffffu, wl[i], m);
    }
  if (tr == 0 && dup * GPL < NG) {
#pragma unroll
    for (int i = 0; i < GPL; ++i) {
      // channels of even index carry C = 16, odd ones C = 256
      zw[((warp * G + pi) * NG + dup * GPL + i) * 2] = zl[i] - 16.f * wl[i];
      zw[((warp * G + pi) * NG + dup * GPL + i) * 2 + 1] = zl[i] - 256.f * wl[i];
    }
  }
  if (owner) {
    mw[(warp * G + pi) * 3 + 0] = mrun;
    mw[(warp * G + pi) * 3 + 1] = lrun;
    mw[(warp * G + pi) * 3 + 2] = erun;
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += NT) {
    const int h = e / D, c = e - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mw[(w * G + h) * 3]);
    float o = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = exp2f(mw[(w * G + h) * 3] - M);
        o = fmaf(f, ow[(w * G + h) * D + c] + zw[((w * G + h) * NG + c / VG) * 2 + (c & 1)], o);
      }
    }
    sc.part_o[(pbase + h) * D + c] = o;
  }
  if (tid < G) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mw[(w * G + tid) * 3]);
    float L = 0.f, E = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = exp2f(mw[(w * G + tid) * 3] - M);
        L = fmaf(f, mw[(w * G + tid) * 3 + 1], L);
        E = fmaf(f, mw[(w * G + tid) * 3 + 2], E);
      }
    }
    sc.part_s[(pbase + tid) * 3 + 0] = M == -INFINITY ? -INFINITY : M * LN2;
    sc.part_s[(pbase + tid) * 3 + 1] = L;
    sc.part_s[(pbase + tid) * 3 + 2] = E;
    sc.part_x[(pbase + tid) * 3 + 0] = 0.5f * S.dmax[tid] * LN2;
    sc.part_x[(pbase + tid) * 3 + 1] = -INFINITY;
    sc.part_x[(pbase + tid) * 3 + 2] = 0.f;
  }
  // ---- the exact residual block (item nb), by the CTA holding it, into partial slot nch ----
  if (do_res) {
    __syncthreads();  // the warps' states above are read: the stage area is free
    const size_t rbase = ((size_t)unit * sc.max_chunks + nch) * G;
    float* lg = reinterpret_cast<float*>(dsm);  // [G][BLK] base-2 logits, then weights
    float* mst = lg + G * BLK;                  // [G][2]
    const int r = rr;
    const __half* kr = t.kres + u * st.res;
    const __half* vr = t.vres + u * st.res;
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
      const float m = nwarp_max(fmaxf(x0, x1));
      const float e0 = lane < r ? exp2f(x0 - m) : 0.f;
      const float e1 = lane + 32 < r ? exp2f(x1 - m) : 0.f;
      const float l = nwarp_sum(e0 + e1);
      lg[h * BLK + lane] = e0;
      lg[h * BLK + lane + 32] = e1;
      if (lane == 0) {
        mst[2 * h] = r > 0 ? m * LN2 : -INFINITY;
        mst[2 * h + 1] = l;
        sc.ell_res[hrow0 + h] = r > 0 ? (m + log2f(l)) * LN2 : -INFINITY;
      }
    }
    __syncthreads();
    for (int c = tid; c < D; c += NT) {
      float o[G];
#pragma unroll
      for (int h = 0; h < G; ++h) o[h] = 0.f;
      for (int tt = 0; tt < r; ++tt) {
        const float v = __half2float(vr[(size_t)tt * D + c]);
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] = fmaf(lg[h * BLK + tt], v, o[h]);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) sc.part_o[(rbase + h) * D + c] = o[h];
    }
    if (tid < G) {
      sc.part_s[(rbase + tid) * 3 + 0] = mst[2 * tid];
      sc.part_s[(rbase + tid) * 3 + 1] = mst[2 * tid + 1];
      sc.part_s[(rbase + tid) * 3 + 2] = 0.f;
      sc.part_x[(rbase + tid) * 3 + 0] = 0.f;
      sc.part_x[(rbase + tid) * 3 + 1] = mst[2 * tid];
      sc.part_x[(rbase + tid) * 3 + 2] = mst[2 * tid + 1];
    }
  }
}

// Split-K combine of the streaming pass, one CTA per (batch row, query head),
// launched as a programmatic dependent of the pass: it is scheduled while the
// pass drains and waits (griddepcontrol.wait) until every CTA of the pass has
// finished and its partials are visible.  The merge itself is merge_parts;
// this kernel adds E_key from the largest Delta and the residual block's mass,
// and E_val = eta mass / L.
template <int D, int G>
__global__ void __launch_bounds__(MERGE_THREADS)
    naive_combine_kernel(DecodeShape sh, Scratch sc, int grid_w, float* __restrict__ out,
                         float* __restrict__ e_key, float* __restrict__ e_val,
                         uint8_t* __restrict__ rung) {
  pdl_begin();
  const int row = blockIdx.x;  // b * Hq + h
  const int b = row / sh.Hq, h = row - b * sh.Hq;
  const int g = h / G, hh = h - g * G;
  const int unit = b * sh.Hkv + g;
  int nb, rr;
  row_blocks(sh, b, nb, rr);
  const int nch = min(grid_w, unit_ctas(sh.sms * NAIVE_CTAS_PER_SM, row_items(nb, rr),
                                        sh.items_sum, naive_cap(nb, sc.max_chunks)));
  const int nparts = nch + 1;  // the last part is the residual block's
  const size_t base = (size_t)unit * sc.max_chunks * G + hh;  // partial index of part 0
  const size_t orow = (size_t)b * sh.Hq + h;
  const MergeStats ms = merge_parts<D, G>(sc, base, nparts, true, out + orow * D);
  if (threadIdx.x == 0) {
    // the residual part holds the residual block's own statistics
    const float* pr = sc.part_x + (base + (size_t)(nparts - 1) * G) * 3;
    const float mr = pr[1];
    const double mres = mr == -INFINITY ? 0.0 : (double)pr[2] * exp((double)mr - ms.M) / ms.L;
    const float ek = nb > 0 ? (float)naive_e_key((double)ms.XA, (double)ms.XA, 1.0 - mres) : 0.f;
    e_key[orow] = ek;
    e_val[orow] = ms.E / ms.L;
    rung[orow] = 0;
    sc.ekey[orow] = ek;
    sc.hflags[orow] = 0;
    sc.kstar[orow] = 0;
    sc.dense[orow] = 0;
  }
}


// Grid width of the streaming pass: the most CTAs any unit receives.  Units
// share sms * 4 CTAs (four resident per SM hold the whole grid in one wave; a
// second wave of even small CTAs measured 25% slower) in proportion to their
// work items; units of shorter rows leave the rest of their grid row
// empty.
int naive_chunks(const DecodeShape& sh, int max_chunks) {
  int w = 1;
  for (int b = 0; b < sh.B; ++b) {
    const int T = sh.lens_host[b], nb = T / BLK, items = row_items(nb, T - nb * BLK);
    const int n = unit_ctas(sh.sms * NAIVE_CTAS_PER_SM, items, sh.items_sum,
                            naive_cap(nb, max_chunks));
    w = n > w ? n : w;
  }
  return w;
}

template <int D, int G, bool MH>
cudaError_t naive_mh(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                     const __half* q, const Scratch& sc, float* out, float* e_key, float* e_val,
                     uint8_t* rung, int trace, cudaStream_t s) {
  const int nch = naive_chunks(sh, sc.max_chunks);
  const int smem = NST * NaiveLayout<D, MH>::STAGE;
  static_assert(NaiveScratchFloats<D, G>::N * 4 <= NST * NaiveLayout<D, false>::STAGE / 2,
                "chunk-end scratch fits the stage area");
  cudaError_t e = ensure_dynamic_smem((const void*)naive_kernel<D, G, MH>, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(naive_kernel<D, G, MH>, dim3(nch, sh.B * sh.Hkv), dim3(NT), smem, s, t, st,
                    unit0, sh, q, sc, trace, out, e_key, e_val, rung);
}

template <int D, int G>
cudaError_t naive_combine_t(const DecodeShape& sh, const Scratch& sc, float* out, float* e_key,
                            float* e_val, uint8_t* rung, cudaStream_t s) {
  const int nch = naive_chunks(sh, sc.max_chunks);
  return launch_pdl(naive_combine_kernel<D, G>, dim3(sh.B * sh.Hq), dim3(MERGE_THREADS), 0, s, sh, sc, nch,
                    out, e_key, e_val, rung);
}

template <int D, int G>
cudaError_t naive_t(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                    const __half* q, const Scratch& sc, float* out, float* e_key, float* e_val,
                    uint8_t* rung, int trace, cudaStream_t s) {
  return t.meta16
             ? naive_mh<D, G, true>(t, st, unit0, sh, q, sc, out, e_key, e_val, rung, trace, s)
             : naive_mh<D, G, false>(t, st, unit0, sh, q, sc, out, e_key, e_val, rung, trace, s);
}

}  // namespace

cudaError_t launch_naive(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                         const __half* q, const Scratch& sc, float* out, float* e_key,
                         float* e_val, uint8_t* rung, int trace, cudaStream_t s) {
#define CQA_NAIVE_CASE(DD, GG) \
  return naive_t<DD, GG>(t, st, unit0, sh, q, sc, out, e_key, e_val, rung, trace, s)
  if (sh.d == 128) {
    switch (sh.G) {
      case 1: CQA_NAIVE_CASE(128, 1);
      case 2: CQA_NAIVE_CASE(128, 2);
      case 4: CQA_NAIVE_CASE(128, 4);
      case 8: CQA_NAIVE_CASE(128, 8);
    }
  } else {
    switch (sh.G) {
      case 1: CQA_NAIVE_CASE(64, 1);
      case 2: CQA_NAIVE_CASE(64, 2);
      case 4: CQA_NAIVE_CASE(64, 4);
    }
  }
#undef CQA_NAIVE_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_naive_combine(const DecodeShape& sh, const Scratch& sc, float* out,
                                 float* e_key, float* e_val, uint8_t* rung, cudaStream_t s) {
#define CQA_NC_CASE(DD, GG) return naive_combine_t<DD, GG>(sh, sc, out, e_key, e_val, rung, s)
  if (sh.d == 128) {
    switch (sh.G) {
      case 1: CQA_NC_CASE(128, 1);
      case 2: CQA_NC_CASE(128, 2);
      case 4: CQA_NC_CASE(128, 4);
      case 8: CQA_NC_CASE(128, 8);
    }
  } else {
    switch (sh.G) {
      case 1: CQA_NC_CASE(64, 1);
      case 2: CQA_NC_CASE(64, 2);
      case 4: CQA_NC_CASE(64, 4);
    }
  }
#undef CQA_NC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace cqa
