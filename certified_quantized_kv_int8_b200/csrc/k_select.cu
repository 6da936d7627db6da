// Coverage selection, rung 1 (widen coverage), key bound E_key and rung 2
// (value promotion), one CTA per (batch row, kv head).
//
// Runtime-Certified Bounded-Error Quantized Attention, Methodology §3
// (adaptive top-K: promote the top-K* blocks covering tau_cov of the
// estimated mass; ladder rung 1 raises K*, rung 2 pages FP16 values for
// blocks whose estimated value-error contribution exceeds v_tol) and §2
// (E_key, a total-variation bound from Delta, computed before any FP16 data
// is touched).
//
// Per query head h of the group:
//   m8_b  = exp(ell8_b - LSE), LSE over all sealed blocks and the exact residual
//   order = blocks by ell8 descending, ties to the lower index (bitonic sort)
//   K*    = fewest leading blocks with m_res + sum m8 >= tau_cov (float64 scan)
// P = union over the group's heads of the selected blocks (their FP16 keys are
// shared).  With T = sealed blocks outside P, dT = max_T Delta, dA = max Delta,
// m8T = sum_T m8:  m_ub = m8T e^dT / (m8T e^dT + (1 - m8T) e^-dA),
//   E_key = min(tanh(dT/2), m_ub (e^(2 dT) - 1)), 0 when T is empty.
// Heads with E_key > eps_key double K* (at most max_expand times).
// A block's FP16 values are promoted when some head has m8_b * eta_b > v_tol.
#include "cqa_internal.cuh"

namespace cqa {

namespace {

constexpr int THREADS = 1024;
constexpr int NWARP = THREADS / 32;

__device__ __forceinline__ uint64_t sort_key(float ell, uint32_t idx) {
  const float f = __fadd_rn(ell, 0.0f);  // one zero
  const uint32_t bits = __float_as_uint(f);
  const uint32_t ord = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
  return ((uint64_t)(~ord) << 32) | idx;  // ascending = ell descending, then index ascending
}

__device__ __forceinline__ float block_max(float x, float* red) {
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = x;
  __syncthreads();
  x = l < NWARP ? red[l] : -INFINITY;
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ double block_sum(double x, double* red) {
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = x;
  __syncthreads();
  x = l < NWARP ? red[l] : 0.0;
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

__device__ __forceinline__ int block_count(int x, int* red) {
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = x;
  __syncthreads();
  x = l < NWARP ? red[l] : 0;
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

__device__ double e_key_bound(double dT, double dA, double m8T) {
  const double a = m8T * exp(dT);
  const double m_ub = a > 0.0 ? a / (a + (1.0 - m8T) * exp(-dA)) : 0.0;
  return fmin(tanh(0.5 * dT), m_ub * expm1(2.0 * dT));
}

// dynamic shared memory: keys u64 [G][NP], mass f32 [G][nb], pflag u8 [nb], vflag u8 [nb]
template <int G>
__global__ void __launch_bounds__(THREADS) select_kernel(Tier1 t, Strides st, int unit0,
                                                         DecodeShape sh, cqa_thresholds th,
                                                         Scratch sc, int NP) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int nb = sh.nb;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem);
  float* mass = reinterpret_cast<float*>(keys + (size_t)G * NP);
  uint8_t* pflag = reinterpret_cast<uint8_t*>(mass + (size_t)G * nb);
  uint8_t* vflag = pflag + nb;
  __shared__ double redd[NWARP];
  __shared__ float redf[NWARP];
  __shared__ int redi[NWARP];
  __shared__ float lse_s[G], mres_s[G], dA_s[G];
  __shared__ int kst[G], kold[G];
  __shared__ double ekey_s[G];
  __shared__ int any_fail;
  __shared__ unsigned hf_s[G];

  const int unit = blockIdx.x;
  const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
  const size_t u = (size_t)unit0 + unit;
  const size_t hrow0 = (size_t)b * sh.Hq + (size_t)g * G;  // first query head of the group
  const float* eta = t.eta + u * st.eta;
  const int tid = threadIdx.x;
  const bool naive = th.naive != 0;

  for (int j = tid; j < nb; j += THREADS) {
    pflag[j] = 0;
    vflag[j] = 0;
  }
  if (tid < G) hf_s[tid] = 0;

  // log-sum-exp per head, masses, Delta max
  for (int h = 0; h < G; ++h) {
    const float* e8 = sc.ell8 + (hrow0 + h) * sh.nbm;
    const float* dl = sc.delta + (hrow0 + h) * sh.nbm;
    const float eres = sc.ell_res[hrow0 + h];
    float mx = eres, dmax = 0.f;
    for (int j = tid; j < nb; j += THREADS) {
      mx = fmaxf(mx, e8[j]);
      dmax = fmaxf(dmax, dl[j]);
    }
    mx = block_max(mx, redf);
    dmax = block_max(dmax, redf);
    double ssum = 0.0;
    for (int j = tid; j < nb; j += THREADS) ssum += (double)expf(e8[j] - mx);
    if (tid == 0 && eres > -INFINITY) ssum += (double)expf(eres - mx);
    ssum = block_sum(ssum, redd);
    const float lse = mx + (float)log(ssum);
    for (int j = tid; j < nb; j += THREADS) mass[h * nb + j] = expf(e8[j] - lse);
    for (int i = tid; i < NP; i += THREADS)
      keys[(size_t)h * NP + i] = i < nb ? sort_key(e8[i], (uint32_t)i) : ~0ull;
    if (tid == 0) {
      lse_s[h] = lse;
      mres_s[h] = eres > -INFINITY ? expf(eres - lse) : 0.f;
      dA_s[h] = dmax;
    }
  }
  __syncthreads();

  // bitonic sort of the G segments of NP keys each
  const int half = NP >> 1;
  for (int k = 2; k <= NP; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int p = tid; p < G * half; p += THREADS) {
        const int seg = p / half, i = p - seg * half;
        const int a = 2 * jj * (i / jj) + (i % jj);
        const int c = a + jj;
        uint64_t* kk = keys + (size_t)seg * NP;
        const uint64_t x = kk[a], y = kk[c];
        const bool up = (a & k) == 0;
        if ((x > y) == up) {
          kk[a] = y;
          kk[c] = x;
        }
      }
      __syncthreads();
    }
  }

  // K* per head: float64 inclusive scan of the sorted masses
  const int per = (nb + THREADS - 1) / THREADS;
  for (int h = 0; h < G; ++h) {
    int kstar = 0;
    if (naive) {
      kstar = 0;
    } else if (th.tau_cov >= 1.0f) {
      kstar = nb;
    } else {
      const double tau = (double)th.tau_cov;
      const double m_res = (double)mres_s[h];
      const uint64_t* kk = keys + (size_t)h * NP;
      const int i0 = tid * per, i1 = min(nb, i0 + per);
      double local = 0.0;
      for (int i = i0; i < i1; ++i) local += (double)mass[h * nb + (int)(kk[i] & 0xffffffffu)];
      // exclusive scan of thread totals
      const int l = tid & 31, w = tid >> 5;
      double incl = local;
      for (int m = 1; m < 32; m <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, m);
        if (l >= m) incl += y;
      }
      __syncthreads();
      if (l == 31) redd[w] = incl;
      __syncthreads();
      double wbase = 0.0;
      for (int x = 0; x < w; ++x) wbase += redd[x];
      double run = m_res + wbase + (incl - local);
      int cnt = 0;
      for (int i = i0; i < i1; ++i) {
        run += (double)mass[h * nb + (int)(kk[i] & 0xffffffffu)];
        cnt += run < tau ? 1 : 0;  // prefix of i + 1 blocks below tau
      }
      cnt = block_count(cnt, redi);
      // prefixes of 0..nb blocks below tau: the empty prefix plus cnt
      kstar = (m_res < tau) ? min(nb, cnt + 1) : 0;
    }
    if (tid == 0) kst[h] = kstar;
    __syncthreads();
  }

  // mark the initial promoted set
  for (int h = 0; h < G; ++h)
    for (int i = tid; i < kst[h]; i += THREADS) pflag[(int)(keys[(size_t)h * NP + i] & 0xffffffffu)] = 1;
  __syncthreads();

  // E_key and rung-1 widening
  for (int round = 0;; ++round) {
    for (int h = 0; h < G; ++h) {
      const float* dl = sc.delta + (hrow0 + h) * sh.nbm;
      float dT = 0.f;
      double m8T = 0.0;
      int ntail = 0;
      for (int j = tid; j < nb; j += THREADS) {
        if (!pflag[j]) {
          dT = fmaxf(dT, dl[j]);
          m8T += (double)mass[h * nb + j];
          ++ntail;
        }
      }
      dT = block_max(dT, redf);
      m8T = block_sum(m8T, redd);
      ntail = block_count(ntail, redi);
      if (tid == 0) ekey_s[h] = ntail ? e_key_bound((double)dT, (double)dA_s[h], m8T) : 0.0;
    }
    __syncthreads();
    if (tid == 0) {
      any_fail = 0;
      for (int h = 0; h < G; ++h) {
        kold[h] = kst[h];
        if (!naive && ekey_s[h] > (double)th.eps_key && round < th.max_expand) {
          kst[h] = min(nb, max(1, 2 * kst[h]));
          hf_s[h] |= HF_WIDENED;
          any_fail = 1;
        }
      }
    }
    __syncthreads();
    if (!any_fail) break;
    for (int h = 0; h < G; ++h)
      for (int i = kold[h] + tid; i < kst[h]; i += THREADS)
        pflag[(int)(keys[(size_t)h * NP + i] & 0xffffffffu)] = 1;
    __syncthreads();
  }

  // rung 2: value promotion
  if (!naive) {
    for (int j = tid; j < nb; j += THREADS) {
      const float e = eta[j];
      uint8_t vp = 0;
      for (int h = 0; h < G; ++h) {
        if (mass[h * nb + j] * e > th.v_tol) {
          vp = 1;
          atomicOr(&hf_s[h], (unsigned)HF_VALUE);
        }
      }
      vflag[j] = vp;
    }
  }
  __syncthreads();

  uint8_t* bf = sc.bflags + ((size_t)b * sh.Hkv + g) * sh.nbm;
  for (int j = tid; j < nb; j += THREADS)
    bf[j] = (pflag[j] ? BF_KEY : 0) | (vflag[j] ? BF_VAL : 0);
  if (tid < G) {
    const int h = tid;
    unsigned f = hf_s[h];
    if (!naive && ekey_s[h] > (double)th.eps_key) f |= HF_KEYFAIL;
    sc.hflags[hrow0 + h] = (uint8_t)f;
    sc.kstar[hrow0 + h] = kst[h];
    sc.ekey[hrow0 + h] = (float)ekey_s[h];
  }
}

template <int G>
cudaError_t launch_select_t(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                            const cqa_thresholds& th, const Scratch& sc, cudaStream_t s) {
  int NP = 2;
  while (NP < sh.nb) NP <<= 1;
  const size_t smem = (size_t)G * NP * 8 + (size_t)G * sh.nb * 4 + 2 * (size_t)sh.nb;
  cudaError_t e = cudaFuncSetAttribute(select_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  select_kernel<G><<<sh.B * sh.Hkv, THREADS, smem, s>>>(t, st, unit0, sh, th, sc, NP);
  return cudaGetLastError();
}

}  // namespace

size_t select_smem_bytes(int G, int nb) {
  int NP = 2;
  while (NP < nb) NP <<= 1;
  return (size_t)G * NP * 8 + (size_t)G * nb * 4 + 2 * (size_t)nb;
}

cudaError_t launch_select(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                          const cqa_thresholds& th, const Scratch& sc, cudaStream_t s) {
  switch (sh.G) {
    case 1: return launch_select_t<1>(t, st, unit0, sh, th, sc, s);
    case 2: return launch_select_t<2>(t, st, unit0, sh, th, sc, s);
    case 4: return launch_select_t<4>(t, st, unit0, sh, th, sc, s);
    case 8: return launch_select_t<8>(t, st, unit0, sh, th, sc, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace cqa
