// The INT8/INT4 decode path with certification off: one streaming pass over
// Tier 1 that scores the INT8 keys, runs the online softmax and accumulates
// the INT4 values, plus a combine that reports E_key and E_val.
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
// codes, key scales, INT4 codes, value scale/offset of one block per stage):
// 14.5 KiB per block for head_dim 128, every byte of Tier 1 read once.
#include "bulk_pipe.cuh"
#include "cqa_internal.cuh"

namespace cqa {

namespace {

constexpr int NT = 128;  // threads per CTA: four warps, four resident CTAs per SM
constexpr int NW = NT / 32;
constexpr int NST = 3;   // stages per CTA

template <int D>
struct NaiveLayout {
  static constexpr int KB = BLK * D;              // INT8 key codes
  static constexpr int SB = 4 * D;                // key scales
  static constexpr int VB = BLK * D / 2;          // INT4 value codes
  static constexpr int MB = BLK * (D / VG) * 8;   // value scale/offset
  static constexpr int STAGE = KB + SB + VB + MB;
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

__device__ __forceinline__ void s8x4_f2(uint32_t w, float2& a, float2& b) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 off = make_float2(-8388736.0f, -8388736.0f);
  a = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)),
                             __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651))), off);
  b = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)),
                             __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653))), off);
}

__device__ __forceinline__ void u4x8_f2(uint32_t w, float2 (&c)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const float2 off = make_float2(-8388608.0f, -8388608.0f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t sel = 0x7650u + (uint32_t)i;
    c[i] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, sel)),
                                  __uint_as_float(__byte_perm(hi, 0x4B000000u, sel))), off);
  }
}

template <int D, int G>
struct NaiveSmem {
  float qf[G][D];        // q * sigma
  float qs[G][D / 16][20];  // q * sigma * key scale of the current block; 16-channel rows
                            // padded to 20 floats so the scoring warps' 16-byte reads
                            // spread over all banks
  float lg[G][BLK];
  float pp[G][BLK];
  float red[NT / (D / 8)][D];
  float m[G], l[G], e[G], alpha[G], dmax[G];
  float mres[G], lres[G];
  float eta[NST];  // eta_b of the block held by each stage
  uint64_t bar[NST];
};

template <int D, int G>
__global__ void __launch_bounds__(NT, 4) naive_kernel(Tier1 t, Strides st, int unit0,
                                                      DecodeShape sh,
                                                      const __half* __restrict__ q, Scratch sc,
                                                      int chunk_blocks, int nres_chunk) {
  using LY = NaiveLayout<D>;
  constexpr int CPT = D / 16;   // lanes per token row in the scoring step (16 channels each)
  constexpr int RPW = 32 / CPT;
  constexpr int LPR = D / 8;    // threads per token row in the P.V step (8 channels each)
  constexpr int RPC = NT / LPR;
  constexpr int NPASS = BLK / RPC;
  constexpr int NG = D / VG;
  constexpr int ROWS_PER_WARP = BLK / NW;  // 16 rows of a block per warp
  constexpr int NLW = ROWS_PER_WARP / RPW;
  static_assert(NLW >= 1, "layout");

  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ NaiveSmem<D, G> S;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.y;
  const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
  const size_t u = (size_t)unit0 + unit;
  const size_t hrow0 = (size_t)b * sh.Hq + (size_t)g * G;
  const int chunk = blockIdx.x;
  const int j0 = chunk * chunk_blocks;
  const int j1 = chunk == nres_chunk ? j0 : min(sh.nb, j0 + chunk_blocks);
  const int nblk = max(0, j1 - j0);

  for (int e = tid; e < G * D; e += NT) {
    const int h = e / D, c = e - h * D;
    S.qf[h][c] = __half2float(q[(hrow0 + h) * D + c]) * sh.sigma;
  }
  if (tid < G) {
    S.m[tid] = -INFINITY;
    S.l[tid] = 0.f;
    S.e[tid] = 0.f;
    S.dmax[tid] = 0.f;
    S.mres[tid] = -INFINITY;
    S.lres[tid] = 0.f;
  }
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
    S.eta[k % NST] = t.eta[u * st.eta + j];  // read by consumers after the stage's barrier
    mbar_arrive_expect_tx(bar, LY::STAGE);
    bulk_g2s(dst, t.kcodes + u * st.kcodes + (size_t)j * LY::KB, LY::KB, bar);
    bulk_g2s(dst + LY::KB, t.kscale + u * st.kscale + (size_t)j * D, LY::SB, bar);
    bulk_g2s(dst + LY::KB + LY::SB, t.vcodes + u * st.vcodes + (size_t)j * LY::VB, LY::VB, bar);
    bulk_g2s(dst + LY::KB + LY::SB + LY::VB, t.vmeta + u * st.vmeta + (size_t)j * BLK * NG * 2,
             LY::MB, bar);
  };
  if (tid == 0)
    for (int k = 0; k < NST; ++k) issue(k);

  const int row = tid / LPR, cl = tid - row * LPR;  // P.V layout
  float2 acc[G][4];
  float zacc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    zacc[h] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[h][i] = make_float2(0.f, 0.f);
  }

  // online-softmax update of head h (warp h) from S.lg[h]; writes S.pp[h]
  auto softmax_step = [&](int h, int ntok, float* ell_out, float eta_b, bool resid) {
    const float x0 = lane < ntok ? S.lg[h][lane] : -INFINITY;
    const float x1 = lane + 32 < ntok ? S.lg[h][lane + 32] : -INFINITY;
    const float mb = nwarp_max(fmaxf(x0, x1));
    const float e0 = expf(x0 - mb), e1 = expf(x1 - mb);
    const float sb = nwarp_sum(e0 + e1);
    const float mold = S.m[h];
    const float mnew = fmaxf(mold, mb);
    const float alpha = mold == -INFINITY ? 0.f : expf(mold - mnew);
    const float c = expf(mb - mnew);
    S.pp[h][lane] = e0 * c;
    S.pp[h][lane + 32] = e1 * c;
    if (lane == 0) {
      const float lb = sb * c;
      S.l[h] = S.l[h] * alpha + lb;
      S.e[h] = S.e[h] * alpha + eta_b * lb;
      S.m[h] = mnew;
      S.alpha[h] = alpha;
      if (ell_out) *ell_out = mb + logf(sb);
      if (resid) {
        S.mres[h] = mb;
        S.lres[h] = sb;
      }
    }
  };

  auto pv_rescale = [&]() {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float al = S.alpha[h];
      zacc[h] *= al;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[h][i].x *= al;
        acc[h][i].y *= al;
      }
    }
  };

  // ---- the exact residual block: a CTA of its own (the last chunk index) ----
  const bool res_cta = chunk == nres_chunk;
  if (res_cta && sh.r > 0) {
    const __half* kr = t.kres + u * st.res;
    const __half* vr = t.vres + u * st.res;
    // LPR threads per token row, 8 channels each; partial dots reduced over the row
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
      const int tt = p * RPC + row;
      float2 kf[4];
      if (tt < sh.r) {
        const uint4 kv = *reinterpret_cast<const uint4*>(kr + (size_t)tt * D + cl * 8);
        const __half2* kh = reinterpret_cast<const __half2*>(&kv);
#pragma unroll
        for (int i = 0; i < 4; ++i) kf[i] = __half22float2(kh[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) kf[i] = make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v = fmaf(S.qf[h][cl * 8 + 2 * i], kf[i].x, v);
          v = fmaf(S.qf[h][cl * 8 + 2 * i + 1], kf[i].y, v);
        }
#pragma unroll
        for (int m = LPR / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
        if (cl == 0) S.lg[h][tt] = tt < sh.r ? v : -INFINITY;
      }
    }
    __syncthreads();
    for (int h = warp; h < G; h += NW) softmax_step(h, sh.r, &sc.ell_res[hrow0 + h], 0.f, true);
    __syncthreads();
    pv_rescale();
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
      const int tt = p * RPC + row;
      if (tt >= sh.r) continue;
      const uint4 vv = *reinterpret_cast<const uint4*>(vr + (size_t)tt * D + cl * 8);
      const __half2* vh = reinterpret_cast<const __half2*>(&vv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 vf = __half22float2(vh[i]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float w = S.pp[h][tt];
          acc[h][i] = __ffma2_rn(make_float2(w, w), vf, acc[h][i]);
        }
      }
    }
    __syncthreads();
  } else if (res_cta && tid < G) {
    sc.ell_res[hrow0 + tid] = -INFINITY;
  }

  // ---- the chunk's sealed blocks ----
  bool ok = true;
  int k = 0;
  const int cc = lane % CPT, tr = lane / CPT;
  for (; k < nblk; ++k) {
    const int j = j0 + k;
    const int stg = k % NST;
    ok = mbar_wait(&S.bar[stg], (uint32_t)((k / NST) & 1), sc.err);
    if (!ok) break;
    const unsigned char* sp = dsm + (size_t)stg * LY::STAGE;
    const uint4* kc = reinterpret_cast<const uint4*>(sp);
    const float* ks = reinterpret_cast<const float*>(sp + LY::KB);
    const uint8_t* vc = sp + LY::KB + LY::SB;
    const float* vm = reinterpret_cast<const float*>(sp + LY::KB + LY::SB + LY::VB);

    // q * sigma * scale, and Delta_b per head (warp h)
    for (int e = tid; e < G * D; e += NT) {
      const int h = e / D, c = e - h * D;
      S.qs[h][c >> 4][c & 15] = S.qf[h][c] * ks[c];
    }
    for (int h = warp; h < G; h += NW) {
      float a = 0.f;
      for (int c = lane; c < D; c += 32) a = fmaf(fabsf(S.qf[h][c]), ks[c], a);
      a = nwarp_sum(a);
      if (lane == 0) {
        const float dl = 0.5f * a;
        S.dmax[h] = fmaxf(S.dmax[h], dl);
        sc.delta[(hrow0 + h) * sh.nbm + j] = dl;
      }
    }
    __syncthreads();

    // INT8 logits: warp w scores rows [w*8, w*8+8)
    {
      float2 qs2[G][8];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4* qp = reinterpret_cast<const float4*>(&S.qs[h][cc][0]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 x = qp[i];
          qs2[h][2 * i] = make_float2(x.x, x.y);
          qs2[h][2 * i + 1] = make_float2(x.z, x.w);
        }
      }
#pragma unroll
      for (int li = 0; li < NLW; ++li) {
        const int r = warp * ROWS_PER_WARP + li * RPW + tr;
        const uint4 ww = kc[r * CPT + cc];
        float2 x[8];
        s8x4_f2(ww.x, x[0], x[1]);
        s8x4_f2(ww.y, x[2], x[3]);
        s8x4_f2(ww.z, x[4], x[5]);
        s8x4_f2(ww.w, x[6], x[7]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float2 a = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 8; ++i) a = __ffma2_rn(qs2[h][i], x[i], a);
          float v = a.x + a.y;
#pragma unroll
          for (int m = CPT / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
          if (cc == 0) S.lg[h][r] = v;
        }
      }
    }
    __syncthreads();
    for (int h = warp; h < G; h += NW)
      softmax_step(h, BLK, &sc.ell8[(hrow0 + h) * sh.nbm + j], S.eta[stg], false);
    if (tid == 0) sc.bflags[(size_t)unit * sh.nbm + j] = 0;  // nothing promoted
    __syncthreads();

    // INT4 P.V with the per-group offset folded
    pv_rescale();
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
      const int tt = p * RPC + row;
      const uint32_t w = *reinterpret_cast<const uint32_t*>(vc + (size_t)tt * (D / 2) + cl * 4);
      const float2 meta = *reinterpret_cast<const float2*>(vm + ((size_t)tt * NG + (cl * 8) / VG) * 2);
      float2 cf[4];
      u4x8_f2(w, cf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pw = S.pp[h][tt];
        const float ws = pw * meta.x;
        zacc[h] = fmaf(pw, meta.y, zacc[h]);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][i] = __ffma2_rn(make_float2(ws, ws), cf[i], acc[h][i]);
      }
    }
    __syncthreads();  // the stage and S.pp are free again
    if (tid == 0) {
      fence_proxy_async_smem();
      issue(k + NST);
    }
  }
  if (!ok) {
    for (int k2 = k + 1; k2 < k + NST && k2 < nblk; ++k2)
      mbar_wait(&S.bar[k2 % NST], (uint32_t)((k2 / NST) & 1), nullptr);
  }

  // ---- partials ----
  const size_t pbase = ((size_t)unit * sc.max_chunks + chunk) * G;
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      S.red[row][cl * 8 + 2 * i] = acc[h][i].x + zacc[h];
      S.red[row][cl * 8 + 2 * i + 1] = acc[h][i].y + zacc[h];
    }
    __syncthreads();
    for (int c = tid; c < D; c += NT) {
      float s = 0.f;
      for (int r = 0; r < RPC; ++r) s += S.red[r][c];
      sc.part_o[(pbase + h) * D + c] = s;
    }
    __syncthreads();
  }
  if (tid < G) {
    sc.part_s[(pbase + tid) * 3 + 0] = S.m[tid];
    sc.part_s[(pbase + tid) * 3 + 1] = S.l[tid];
    sc.part_s[(pbase + tid) * 3 + 2] = S.e[tid];
    sc.part_x[(pbase + tid) * 3 + 0] = S.dmax[tid];
    sc.part_x[(pbase + tid) * 3 + 1] = S.mres[tid];
    sc.part_x[(pbase + tid) * 3 + 2] = S.lres[tid];
  }
}

__device__ double naive_e_key(double dT, double dA, double m8T) {
  const double a = m8T * exp(dT);
  const double m_ub = a > 0.0 ? a / (a + (1.0 - m8T) * exp(-dA)) : 0.0;
  return fmin(tanh(0.5 * dT), m_ub * expm1(2.0 * dT));
}

// one CTA of D threads per (batch row, query head); thread c owns output channel c
template <int D, int G>
__global__ void naive_combine_kernel(DecodeShape sh, Scratch sc, int nchunks, int res_chunk,
                                     float* __restrict__ out, float* __restrict__ e_key,
                                     float* __restrict__ e_val, uint8_t* __restrict__ rung) {
  constexpr int NW = D / 32;
  __shared__ float wbuf[1024];
  __shared__ float red[3][NW];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  const int b = row / sh.Hq, h = row - b * sh.Hq;
  const int g = h / G, hh = h - g * G;
  const int unit = b * sh.Hkv + g;
  const size_t base = (size_t)unit * sc.max_chunks * G + hh;
  float ml = -INFINITY, dl = 0.f;
  for (int c = tid; c < nchunks; c += D) {
    ml = fmaxf(ml, sc.part_s[(base + (size_t)c * G) * 3]);
    dl = fmaxf(dl, sc.part_x[(base + (size_t)c * G) * 3]);
  }
  ml = nwarp_max(ml);
  dl = nwarp_max(dl);
  if (lane == 0) {
    red[0][warp] = ml;
    red[1][warp] = dl;
  }
  __syncthreads();
  float M = -INFINITY, dA = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    M = fmaxf(M, red[0][w]);
    dA = fmaxf(dA, red[1][w]);
  }
  __syncthreads();
  float ll = 0.f, el = 0.f;
  for (int c = tid; c < nchunks; c += D) {
    const float* ps = sc.part_s + (base + (size_t)c * G) * 3;
    const float w = ps[0] == -INFINITY ? 0.f : expf(ps[0] - M);
    if (c < 1024) wbuf[c] = w;
    ll += ps[1] * w;
    el += ps[2] * w;
  }
  ll = nwarp_sum(ll);
  el = nwarp_sum(el);
  if (lane == 0) {
    red[0][warp] = ll;
    red[1][warp] = el;
  }
  __syncthreads();
  float L = 0.f, E = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    L += red[0][w];
    E += red[1][w];
  }
  // o: batches of 16 independent loads so the chain of chunk partials does not
  // serialise on memory latency
  float o = 0.f;
  for (int c0 = 0; c0 < nchunks; c0 += 16) {
    float v[16], wv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = c0 + i;
      v[i] = 0.f;
      wv[i] = 0.f;
      if (c < nchunks) {
        const size_t pi = base + (size_t)c * G;
        v[i] = sc.part_o[pi * D + tid];
        if (c < 1024) {
          wv[i] = wbuf[c];
        } else {
          const float mc = sc.part_s[pi * 3];
          wv[i] = mc == -INFINITY ? 0.f : expf(mc - M);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) o = fmaf(v[i], wv[i], o);
  }
  out[(size_t)row * D + tid] = o / L;
  if (tid == 0) {
    // the residual CTA holds the residual's own statistics
    const float* px = sc.part_x + (base + (size_t)res_chunk * G) * 3;
    const double mres = px[1] == -INFINITY ? 0.0 : (double)px[2] * exp((double)px[1] - M) / L;
    const double m8T = 1.0 - mres;
    const float ek = sh.nb > 0 ? (float)naive_e_key((double)dA, (double)dA, m8T) : 0.f;
    e_key[row] = ek;
    e_val[row] = E / L;
    rung[row] = 0;
    sc.ekey[row] = ek;
    sc.hflags[row] = 0;
    sc.kstar[row] = 0;
    sc.dense[row] = 0;
  }
}

// chunking of the streaming pass: about four resident CTAs per SM over all units
void naive_chunking(const DecodeShape& sh, int max_chunks, int* cb, int* nch) {
  const int units = sh.B * sh.Hkv;
  int per_unit = (148 * 4 + units - 1) / units;
  if (per_unit > max_chunks - 1) per_unit = max_chunks - 1;  // one partial slot for the residual
  if (per_unit < 1) per_unit = 1;
  int c = sh.nb > 0 ? (sh.nb + per_unit - 1) / per_unit : 1;
  if (c < 1) c = 1;
  int n = sh.nb > 0 ? (sh.nb + c - 1) / c : 1;
  *cb = c;
  *nch = n < 1 ? 1 : n;
}

template <int D, int G>
cudaError_t naive_t(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                    const __half* q, const Scratch& sc, float* out, float* e_key, float* e_val,
                    uint8_t* rung, int part, cudaStream_t s) {
  int cb, nch;
  naive_chunking(sh, sc.max_chunks, &cb, &nch);
  if (part == 0) {
    const int smem = NST * NaiveLayout<D>::STAGE;
    cudaError_t e = ensure_dynamic_smem((const void*)naive_kernel<D, G>, (int)smem);
    if (e != cudaSuccess) return e;
    naive_kernel<D, G><<<dim3(nch + 1, sh.B * sh.Hkv), NT, smem, s>>>(t, st, unit0, sh, q, sc,
                                                                      cb, nch);
    return cudaGetLastError();
  }
  naive_combine_kernel<D, G><<<sh.B * sh.Hq, D, 0, s>>>(sh, sc, nch + 1, nch, out, e_key, e_val,
                                                          rung);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_naive(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                         const __half* q, const Scratch& sc, float* out, float* e_key,
                         float* e_val, uint8_t* rung, int part, cudaStream_t s) {
#define CQA_NAIVE_CASE(DD, GG) \
  return naive_t<DD, GG>(t, st, unit0, sh, q, sc, out, e_key, e_val, rung, part, s)
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

}  // namespace cqa
