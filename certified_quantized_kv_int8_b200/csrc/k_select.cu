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
//
// Two kernels.  Rows of up to 256 sealed blocks: one warp per query head holds
// the head's blocks, sort keys and scan in registers (select_small_kernel).
// Longer rows: the CTA's 1024 threads form G groups, one per query head; the
// per-head work (log-sum-exp, sort, scan, tail reductions) synchronises each
// group on its own named barrier, and only the union steps use the whole CTA
// (select_kernel).
#include "cqa_internal.cuh"

namespace cqa {

namespace {

constexpr int THREADS = 1024;

__device__ __forceinline__ uint64_t sort_key(float ell, uint32_t idx) {
  const float f = __fadd_rn(ell, 0.0f);  // one zero
  const uint32_t bits = __float_as_uint(f);
  const uint32_t ord = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
  return ((uint64_t)(~ord) << 32) | idx;  // ascending = ell descending, then index ascending
}

__device__ __forceinline__ void group_bar(int grp, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(grp + 1), "r"(nthreads) : "memory");
}

template <class T>
__device__ __forceinline__ T wmax(T x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
    const T y = __shfl_xor_sync(0xffffffffu, x, m);
    x = x > y ? x : y;
  }
  return x;
}

template <class T>
__device__ __forceinline__ T wsum(T x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// Reductions over one thread group (nw warps) through a per-group slot array.
struct Group {
  int id, nthreads, nw, wig, lane, tig;
  template <class T>
  __device__ T max(T x, T* slot, T ident) const {
    x = wmax(x);
    group_bar(id, nthreads);
    if (lane == 0) slot[wig] = x;
    group_bar(id, nthreads);
    x = lane < nw ? slot[lane] : ident;
    return wmax(x);
  }
  template <class T>
  __device__ T sum(T x, T* slot) const {
    x = wsum(x);
    group_bar(id, nthreads);
    if (lane == 0) slot[wig] = x;
    group_bar(id, nthreads);
    x = lane < nw ? slot[lane] : T(0);
    return wsum(x);
  }
  __device__ void sync() const { group_bar(id, nthreads); }
};

// Bitonic sort (ascending) of one head's keys by its GT-thread group, E keys per
// thread in registers: thread tg holds positions tg*E .. tg*E + E - 1.  Distances
// below E are swaps inside a thread, below 32*E shuffles inside a warp; only the
// widest stages exchange through shared memory (x, E*GT keys, laid out [r][tg] so
// a warp's accesses are consecutive).  On entry keys[0, E*GT) holds the keys; on
// exit it holds them sorted.
template <int E>
__device__ void group_sort(uint64_t* keys, int tg, int GT, const Group& grp) {
  uint64_t v[E];
#pragma unroll
  for (int r = 0; r < E; ++r) v[r] = keys[tg * E + r];
  grp.sync();  // every thread has its keys: the array is free for the exchanges
  const int n = GT * E;
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < E) {
#pragma unroll
        for (int jj = E / 2; jj >= 1; jj >>= 1) {
          if (jj == j) {
#pragma unroll
            for (int r = 0; r < E; ++r) {
              if ((r & jj) == 0) {
                const bool up = ((tg * E + r) & k) == 0;
                const uint64_t a = v[r], b = v[r + jj];
                if ((a > b) == up) {
                  v[r] = b;
                  v[r + jj] = a;
                }
              }
            }
          }
        }
      } else {
        const int m = j / E;  // distance in threads
        const bool keep_min = ((tg & m) == 0) == (((tg * E) & k) == 0);
        if (m < 32) {
#pragma unroll
          for (int r = 0; r < E; ++r) {
            const uint64_t o = __shfl_xor_sync(0xffffffffu, v[r], m);
            v[r] = keep_min ? (o < v[r] ? o : v[r]) : (o > v[r] ? o : v[r]);
          }
        } else {
#pragma unroll
          for (int r = 0; r < E; ++r) keys[r * GT + tg] = v[r];
          grp.sync();
#pragma unroll
          for (int r = 0; r < E; ++r) {
            const uint64_t o = keys[r * GT + (tg ^ m)];
            v[r] = keep_min ? (o < v[r] ? o : v[r]) : (o > v[r] ? o : v[r]);
          }
          grp.sync();
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < E; ++r) keys[tg * E + r] = v[r];
  grp.sync();
}

__device__ double e_key_bound(double dT, double dA, double m8T) {
  const double a = m8T * exp(dT);
  const double m_ub = a > 0.0 ? a / (a + (1.0 - m8T) * exp(-dA)) : 0.0;
  return fmin(tanh(0.5 * dT), m_ub * expm1(2.0 * dT));
}

// dynamic shared memory, sized for the longest row (nbL = nb_max blocks):
// keys u64 [G][NP], mass f32 [G][nbL], pflag u8 [nbL], vflag u8 [nbL]
template <int G>
__global__ void __launch_bounds__(THREADS) select_kernel(Tier1 t, Strides st, int unit0,
                                                         DecodeShape sh, cqa_thresholds th,
                                                         Scratch sc, int NP) {
  pdl_begin();
  extern __shared__ __align__(16) unsigned char smem[];
  const int nbL = sh.nb_max;
  uint64_t* keys_all = reinterpret_cast<uint64_t*>(smem);
  float* mass_all = reinterpret_cast<float*>(keys_all + (size_t)G * NP);
  uint8_t* pflag = reinterpret_cast<uint8_t*>(mass_all + (size_t)G * nbL);
  uint8_t* vflag = pflag + nbL;
  constexpr int GT = THREADS / G;  // threads per head group
  __shared__ double slot_d[G][32];
  __shared__ float slot_f[G][32];
  __shared__ int slot_i[G][32];
  __shared__ int kst[G], kold[G];
  __shared__ double ekey_s[G];
  __shared__ int any_fail;
  __shared__ int npro_s;
  __shared__ unsigned hf_s[G];

  const int unit = blockIdx.x;
  const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
  const size_t u = (size_t)unit0 + unit;
  const size_t hrow0 = (size_t)b * sh.Hq + (size_t)g * G;
  const int tid = threadIdx.x;
  const bool naive = th.naive != 0;
  int nb, r_unused;  // this row's sealed blocks (at most nbL)
  row_blocks(sh, b, nb, r_unused);
  Group grp;
  grp.id = tid / GT;
  grp.nthreads = GT;
  grp.nw = GT / 32;
  grp.tig = tid - grp.id * GT;
  grp.wig = grp.tig >> 5;
  grp.lane = tid & 31;
  const int h = grp.id;  // this group's head
  const int tg = grp.tig;
  uint64_t* keys = keys_all + (size_t)h * NP;
  float* mass = mass_all + (size_t)h * nbL;
  const float* e8 = sc.ell8 + (hrow0 + h) * sh.nbm;
  const float* dl = sc.delta + (hrow0 + h) * sh.nbm;

  for (int j = tid; j < nb; j += THREADS) {
    pflag[j] = 0;
    vflag[j] = 0;
  }
  if (tid < G) hf_s[tid] = 0;
  if (tid == 0) npro_s = 0;

  // ---- per head: log-sum-exp, masses, Delta max, sort keys ----
  const float eres = sc.ell_res[hrow0 + h];
  float mx = eres, dmax = 0.f;
  for (int j = tg; j < nb; j += GT) {
    mx = fmaxf(mx, e8[j]);
    dmax = fmaxf(dmax, dl[j]);
  }
  mx = grp.max(mx, slot_f[h], -INFINITY);
  const float dA = grp.max(dmax, slot_f[h], 0.f);
  double ssum = 0.0;
  for (int j = tg; j < nb; j += GT) ssum += (double)expf(e8[j] - mx);
  if (tg == 0 && eres > -INFINITY) ssum += (double)expf(eres - mx);
  ssum = grp.sum(ssum, slot_d[h]);
  const float lse = mx + (float)log(ssum);
  for (int j = tg; j < nb; j += GT) mass[j] = expf(e8[j] - lse);
  for (int i = tg; i < NP; i += GT) keys[i] = i < nb ? sort_key(e8[i], (uint32_t)i) : ~0ull;
  const float m_res_f = eres > -INFINITY ? expf(eres - lse) : 0.f;
  grp.sync();

  // ---- bitonic sort of this head's NP keys ----
  // NP keys padded with sentinels to E = NP / GT >= 1 keys per thread (registers,
  // up to 8 within the 64 registers a thread has at 1024 threads per CTA)
  const int Ek = NP > GT ? NP / GT : 1;
  switch (Ek) {
    case 1: group_sort<1>(keys, tg, GT, grp); break;
    case 2: group_sort<2>(keys, tg, GT, grp); break;
    case 4: group_sort<4>(keys, tg, GT, grp); break;
    case 8: group_sort<8>(keys, tg, GT, grp); break;
    default: break;
  }
  const int half = NP >> 1;
  for (int k = 2; Ek > 8 && k <= NP; k <<= 1) {  // longer heads: in shared memory
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int p = tg; p < half; p += GT) {
        const int a = 2 * jj * (p / jj) + (p % jj);
        const int c = a + jj;
        const uint64_t x = keys[a], y = keys[c];
        const bool up = (a & k) == 0;
        if ((x > y) == up) {
          keys[a] = y;
          keys[c] = x;
        }
      }
      grp.sync();
    }
  }

  // ---- K*: float64 inclusive scan of the sorted masses ----
  int kstar = 0;
  if (naive) {
    kstar = 0;
  } else if (th.tau_cov >= 1.0f) {
    kstar = nb;
  } else {
    const double tau = (double)th.tau_cov;
    const double m_res = (double)m_res_f;
    const int per = (nb + GT - 1) / GT;
    const int i0 = tg * per, i1 = min(nb, i0 + per);
    double local = 0.0;
    for (int i = i0; i < i1; ++i) local += (double)mass[(int)(keys[i] & 0xffffffffu)];
    double incl = local;
    for (int m = 1; m < 32; m <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, m);
      if (grp.lane >= m) incl += y;
    }
    grp.sync();
    if (grp.lane == 31) slot_d[h][grp.wig] = incl;
    grp.sync();
    double wbase = 0.0;
    for (int x = 0; x < grp.wig; ++x) wbase += slot_d[h][x];
    double run = m_res + wbase + (incl - local);
    int cnt = 0;
    for (int i = i0; i < i1; ++i) {
      run += (double)mass[(int)(keys[i] & 0xffffffffu)];
      cnt += run < tau ? 1 : 0;  // prefix of i + 1 blocks below tau
    }
    cnt = grp.sum(cnt, slot_i[h]);
    // prefixes of 0..nb blocks below tau: the empty prefix plus cnt
    kstar = (m_res < tau) ? min(nb, cnt + 1) : 0;
  }
  if (tg == 0) kst[h] = kstar;
  for (int i = tg; i < kstar; i += GT) pflag[(int)(keys[i] & 0xffffffffu)] = 1;
  __syncthreads();

  // ---- E_key and rung-1 widening ----
  for (int round = 0;; ++round) {
    float dT = 0.f;
    double m8T = 0.0;
    int ntail = 0;
    for (int j = tg; j < nb; j += GT) {
      if (!pflag[j]) {
        dT = fmaxf(dT, dl[j]);
        m8T += (double)mass[j];
        ++ntail;
      }
    }
    dT = grp.max(dT, slot_f[h], 0.f);
    m8T = grp.sum(m8T, slot_d[h]);
    ntail = grp.sum(ntail, slot_i[h]);
    if (tg == 0) ekey_s[h] = ntail ? e_key_bound((double)dT, (double)dA, m8T) : 0.0;
    __syncthreads();
    if (tid == 0) {
      any_fail = 0;
      for (int hh = 0; hh < G; ++hh) {
        kold[hh] = kst[hh];
        if (!naive && ekey_s[hh] > (double)th.eps_key && round < th.max_expand) {
          kst[hh] = min(nb, max(1, 2 * kst[hh]));
          hf_s[hh] |= HF_WIDENED;
          any_fail = 1;
        }
      }
    }
    __syncthreads();
    if (!any_fail) break;
    for (int i = kold[h] + tg; i < kst[h]; i += GT) pflag[(int)(keys[i] & 0xffffffffu)] = 1;
    __syncthreads();
  }

  // ---- rung 2: value promotion ----
  const float* eta = t.eta + u * st.eta;
  if (!naive) {
    for (int j = tid; j < nb; j += THREADS) {
      const float e = eta[j];
      uint8_t vp = 0;
      for (int hh = 0; hh < G; ++hh) {
        if (mass_all[(size_t)hh * nbL + j] * e > th.v_tol) {
          vp = 1;
          atomicOr(&hf_s[hh], (unsigned)HF_VALUE);
        }
      }
      vflag[j] = vp;
    }
  }
  __syncthreads();

  uint8_t* bf = sc.bflags + ((size_t)b * sh.Hkv + g) * sh.nbm;
  int npro = 0;
  for (int j = tid; j < nb; j += THREADS) {
    bf[j] = (pflag[j] ? BF_KEY : 0) | (vflag[j] ? BF_VAL : 0);
    npro += pflag[j] ? 1 : 0;
  }
  // promoted-block count of the unit, for the host's key-prefetch policy
  npro = wsum(npro);
  if (grp.lane == 0 && npro) atomicAdd(&npro_s, npro);
  __syncthreads();
  if (tid == 0 && sc.promo) sc.promo[u] = npro_s;
  if (tid < G) {
    const int hh = tid;
    unsigned f = hf_s[hh];
    if (!naive && ekey_s[hh] > (double)th.eps_key) f |= HF_KEYFAIL;
    sc.hflags[hrow0 + hh] = (uint8_t)f;
    sc.kstar[hrow0 + hh] = kst[hh];
    sc.ekey[hrow0 + hh] = (float)ekey_s[hh];
  }
}

// Bitonic sort (ascending) of 32 * E keys by one warp, E keys per lane in
// registers (lane l holds positions l*E .. l*E + E - 1 on exit): distances
// below E are swaps inside a lane, the rest shuffles; no shared memory and no
// barrier.
template <int E>
__device__ __forceinline__ void warp_sort(uint64_t (&v)[E], int lane) {
  constexpr int n = 32 * E;
#pragma unroll
  for (int k = 2; k <= n; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < E) {
#pragma unroll
        for (int r = 0; r < E; ++r) {
          if ((r & j) == 0) {
            const bool up = ((lane * E + r) & k) == 0;
            const uint64_t a = v[r], b = v[r + j];
            if ((a > b) == up) {
              v[r] = b;
              v[r + j] = a;
            }
          }
        }
      } else {
        const int m = j / E;  // distance in lanes
        const bool keep_min = ((lane & m) == 0) == (((lane * E) & k) == 0);
#pragma unroll
        for (int r = 0; r < E; ++r) {
          const uint64_t o = __shfl_xor_sync(0xffffffffu, v[r], m);
          v[r] = keep_min ? (o < v[r] ? o : v[r]) : (o > v[r] ? o : v[r]);
        }
      }
    }
  }
}

// The same selection for rows of at most 32 * E <= 256 sealed blocks (contexts
// up to 16K tokens), where the 1024-thread kernel's named barriers set its
// time: one warp per query head, the head's blocks in registers (E per lane),
// its reductions, sort and K* scan done with shuffles; the CTA synchronises
// only for the union P, the widening rounds and value promotion.  Same
// quantities, same float64 scan, same tie order as select_kernel.
template <int G, int E>
__global__ void __launch_bounds__(32 * G) select_small_kernel(Tier1 t, Strides st, int unit0,
                                                              DecodeShape sh, cqa_thresholds th,
                                                              Scratch sc) {
  pdl_begin();
  constexpr int NP = 32 * E;
  constexpr int NT = 32 * G;
  __shared__ float mass_all[G][NP];
  __shared__ uint8_t pflag[NP], vflag[NP];
  __shared__ int kst[G], kold[G];
  __shared__ double ekey_s[G];
  __shared__ int any_fail;
  __shared__ int npro_s;
  __shared__ unsigned hf_s[G];

  const int unit = blockIdx.x;
  const int b = unit / sh.Hkv, g = unit - b * sh.Hkv;
  const size_t u = (size_t)unit0 + unit;
  const size_t hrow0 = (size_t)b * sh.Hq + (size_t)g * G;
  const int tid = threadIdx.x, h = tid >> 5, lane = tid & 31;
  const bool naive = th.naive != 0;
  int nb, r_unused;  // this row's sealed blocks (at most NP)
  row_blocks(sh, b, nb, r_unused);
  const float* e8 = sc.ell8 + (hrow0 + h) * sh.nbm;
  const float* dl = sc.delta + (hrow0 + h) * sh.nbm;

  for (int j = tid; j < NP; j += NT) {
    pflag[j] = 0;
    vflag[j] = 0;
  }
  if (tid < G) hf_s[tid] = 0;
  if (tid == 0) npro_s = 0;

  // eta_b of the blocks this thread checks for value promotion, loaded with the keys
  constexpr int NE = (NP + NT - 1) / NT;
  const float* eta = t.eta + u * st.eta;
  float etv[NE];
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int j = tid + i * NT;
    etv[i] = (!naive && j < nb) ? eta[j] : 0.f;
  }

  // ---- per head: log-sum-exp, masses, Delta max; lane holds blocks lane + 32 i ----
  const float eres = sc.ell_res[hrow0 + h];
  float ev[E], dv[E], ms[E];
  float mx = eres, dmax = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int j = lane + 32 * i;
    ev[i] = j < nb ? e8[j] : -INFINITY;
    dv[i] = j < nb ? dl[j] : 0.f;
    mx = fmaxf(mx, ev[i]);
    dmax = fmaxf(dmax, dv[i]);
  }
  mx = wmax(mx);
  const float dA = wmax(dmax);
  double ssum = 0.0;
#pragma unroll
  for (int i = 0; i < E; ++i)
    if (lane + 32 * i < nb) ssum += (double)expf(ev[i] - mx);
  if (lane == 0 && eres > -INFINITY) ssum += (double)expf(eres - mx);
  ssum = wsum(ssum);
  const float lse = mx + (float)log(ssum);
  uint64_t v[E];  // sort keys; any starting arrangement sorts to the same order
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int j = lane + 32 * i;
    ms[i] = j < nb ? expf(ev[i] - lse) : 0.f;
    mass_all[h][j] = ms[i];
    v[i] = j < nb ? sort_key(ev[i], (uint32_t)j) : ~0ull;
  }
  const float m_res_f = eres > -INFINITY ? expf(eres - lse) : 0.f;
  warp_sort<E>(v, lane);  // now position lane * E + r
  __syncwarp();           // the head's masses are in shared memory

  // ---- K*: float64 inclusive scan of the sorted masses ----
  int kstar = 0;
  if (naive) {
    kstar = 0;
  } else if (th.tau_cov >= 1.0f) {
    kstar = nb;
  } else {
    const double tau = (double)th.tau_cov;
    const double m_res = (double)m_res_f;
    double mr[E], local = 0.0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const int p = lane * E + r;
      mr[r] = p < nb ? (double)mass_all[h][(int)(v[r] & 0xffffffffu)] : 0.0;
      local += mr[r];
    }
    double incl = local;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, m);
      if (lane >= m) incl += y;
    }
    double run = m_res + (incl - local);
    int cnt = 0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      if (lane * E + r < nb) {
        run += mr[r];
        cnt += run < tau ? 1 : 0;  // prefix of position + 1 blocks below tau
      }
    }
    cnt = wsum(cnt);
    kstar = (m_res < tau) ? min(nb, cnt + 1) : 0;
  }
  if (lane == 0) kst[h] = kstar;
#pragma unroll
  for (int r = 0; r < E; ++r)
    if (lane * E + r < kstar) pflag[(int)(v[r] & 0xffffffffu)] = 1;
  __syncthreads();

  // ---- E_key and rung-1 widening ----
  for (int round = 0;; ++round) {
    float dT = 0.f;
    double m8T = 0.0;
    int ntail = 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const int j = lane + 32 * i;
      if (j < nb && !pflag[j]) {
        dT = fmaxf(dT, dv[i]);
        m8T += (double)ms[i];
        ++ntail;
      }
    }
    dT = wmax(dT);
    m8T = wsum(m8T);
    ntail = wsum(ntail);
    if (lane == 0) ekey_s[h] = ntail ? e_key_bound((double)dT, (double)dA, m8T) : 0.0;
    __syncthreads();
    if (tid == 0) {
      any_fail = 0;
      for (int hh = 0; hh < G; ++hh) {
        kold[hh] = kst[hh];
        if (!naive && ekey_s[hh] > (double)th.eps_key && round < th.max_expand) {
          kst[hh] = min(nb, max(1, 2 * kst[hh]));
          hf_s[hh] |= HF_WIDENED;
          any_fail = 1;
        }
      }
    }
    __syncthreads();
    if (!any_fail) break;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const int p = lane * E + r;
      if (p >= kold[h] && p < kst[h]) pflag[(int)(v[r] & 0xffffffffu)] = 1;
    }
    __syncthreads();
  }

  // ---- rung 2: value promotion ----
  if (!naive) {
#pragma unroll
    for (int i = 0; i < NE; ++i) {
      const int j = tid + i * NT;
      if (j >= nb) continue;
      const float e = etv[i];
      uint8_t vp = 0;
      for (int hh = 0; hh < G; ++hh) {
        if (mass_all[hh][j] * e > th.v_tol) {
          vp = 1;
          atomicOr(&hf_s[hh], (unsigned)HF_VALUE);
        }
      }
      vflag[j] = vp;
    }
  }
  __syncthreads();

  uint8_t* bf = sc.bflags + ((size_t)b * sh.Hkv + g) * sh.nbm;
  int npro = 0;
  for (int j = tid; j < nb; j += NT) {
    bf[j] = (pflag[j] ? BF_KEY : 0) | (vflag[j] ? BF_VAL : 0);
    npro += pflag[j] ? 1 : 0;
  }
  npro = wsum(npro);
  if (lane == 0 && npro) atomicAdd(&npro_s, npro);
  __syncthreads();
  if (tid == 0 && sc.promo) sc.promo[u] = npro_s;
  if (tid < G) {
    const int hh = tid;
    unsigned f = hf_s[hh];
    if (!naive && ekey_s[hh] > (double)th.eps_key) f |= HF_KEYFAIL;
    sc.hflags[hrow0 + hh] = (uint8_t)f;
    sc.kstar[hrow0 + hh] = kst[hh];
    sc.ekey[hrow0 + hh] = (float)ekey_s[hh];
  }
}

template <int G>
cudaError_t launch_select_t(const Tier1& t, const Strides& st, int unit0, const DecodeShape& sh,
                            const cqa_thresholds& th, const Scratch& sc, cudaStream_t s) {
  if (sh.nb_max <= 256) {  // one warp per head, keys in registers
    const dim3 grid(sh.B * sh.Hkv), block(32 * G);
    if (sh.nb_max <= 32)
      return launch_pdl(select_small_kernel<G, 1>, grid, block, 0, s, t, st, unit0, sh, th, sc);
    if (sh.nb_max <= 64)
      return launch_pdl(select_small_kernel<G, 2>, grid, block, 0, s, t, st, unit0, sh, th, sc);
    if (sh.nb_max <= 128)
      return launch_pdl(select_small_kernel<G, 4>, grid, block, 0, s, t, st, unit0, sh, th, sc);
    return launch_pdl(select_small_kernel<G, 8>, grid, block, 0, s, t, st, unit0, sh, th, sc);
  }
  int NP = 2;
  while (NP < sh.nb_max) NP <<= 1;
  if (NP < THREADS / G) NP = THREADS / G;  // at least one key per thread of a head group
  const size_t smem = (size_t)G * NP * 8 + (size_t)G * sh.nb_max * 4 + 2 * (size_t)sh.nb_max;
  cudaError_t e = ensure_dynamic_smem((const void*)select_kernel<G>, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(select_kernel<G>, dim3(sh.B * sh.Hkv), dim3(THREADS), smem, s, t, st, unit0, sh,
                    th, sc, NP);
}

}  // namespace

size_t select_smem_bytes(int G, int nb) {
  int NP = 2;
  while (NP < nb) NP <<= 1;
  if (NP < THREADS / G) NP = THREADS / G;
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
