// Block-ranking consistency check with the rung 3 / rung 4 decisions (before
// the attention pass), split-K combine with the value bound E_val (after it),
// and the combine of the dense passes from Tier 2.
//
// Runtime-Certified Bounded-Error Quantized Attention, Methodology §2
// (E_val = sum over INT4-valued blocks of attention mass times eta_b) and §3
// (rank-consistency check: the INT8 ranking of the promoted blocks is compared
// with their FP16 ranking, a mismatch sends the head to dense attention;
// rung 4 recomputes the whole layer densely).
//
// Readings used: the check takes the top-min(rank_r, |P|) promoted blocks by
// INT8 and by FP16 block log-mass (each ordered by log-mass descending, ties
// to the lower block index) and counts the pairs of the union of the two lists
// that the two rankings order the other way round; more than rank_tol such
// pairs is a failure (rank_tol = 0: the ordered lists must be equal).  Rung 3
// also fires when E_key stayed above eps_key after widening; rung 4 fires when
// at least need_dense = ceil(layer_dense_frac * n_q_heads) heads of a (layer,
// batch row) took rung 3 that way.  After the attention pass, a head whose
// E_val exceeds eps_val also takes rung 3 (post-check, not counted for rung 4).
#include "cqa_internal.cuh"
#include "split_merge.cuh"

namespace cqa {

namespace {

struct KI {
  float k;
  int i;
};

// (key descending, index ascending): true when a comes before b
__device__ __forceinline__ bool before(KI a, KI b) { return a.k > b.k || (a.k == b.k && a.i < b.i); }

// Rank check and the rung 3 / rung 4 decision, before the attention pass.
// One warp per (batch row, query head), DWH heads per CTA; no CTA barrier.
// The two top-r lists are built one rank at a time by warp-wide arg-bests
// under the (key desc, index asc) orders, over the head's promoted blocks held
// in registers (E per lane: rows of at most 32 * E <= 256 blocks); their union
// U (at most 2 * MAX_RANK_R blocks) is then compared pair by pair.  The last head of a batch row to finish takes the
// whole-layer decision (rung 4).
constexpr int DWH = 8;  // heads (warps) per CTA

__device__ __forceinline__ KI ki_best(KI a, KI b) { return before(b, a) ? b : a; }

__device__ __forceinline__ KI warp_best(KI v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
    KI o;
    o.k = __shfl_xor_sync(0xffffffffu, v.k, m);
    o.i = __shfl_xor_sync(0xffffffffu, v.i, m);
    v = ki_best(v, o);
  }
  return v;
}

template <int E>
__global__ void __launch_bounds__(32 * DWH) decide_kernel(DecodeShape sh, cqa_thresholds th,
                                                          int need_dense, Scratch sc) {
  pdl_begin();
  __shared__ int top8[DWH][MAX_RANK_R], top16[DWH][MAX_RANK_R];
  __shared__ int uni[DWH][2 * MAX_RANK_R];
  __shared__ float u8[DWH][2 * MAX_RANK_R], u16[DWH][2 * MAX_RANK_R];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int row_i = blockIdx.x * DWH + w;  // b * Hq + h
  if (row_i >= sh.B * sh.Hq) return;       // the whole warp: nothing below waits on it
  const int b = row_i / sh.Hq, h = row_i - b * sh.Hq;
  const int unit = b * sh.Hkv + h / sh.G;
  const size_t row = (size_t)row_i;
  int nb, r_unused;  // this batch row's sealed blocks
  row_blocks(sh, b, nb, r_unused);
  const uint8_t* bf = sc.bflags + (size_t)unit * sh.nbm;
  const float* e8 = sc.ell8 + row * sh.nbm;
  const float* e16 = sc.ell16 + row * sh.nbm;
  static_assert(E >= 1 && E <= 8, "rows of at most 256 blocks");
  const uint8_t hf0 = lane == 0 ? sc.hflags[row] : (uint8_t)0;  // loaded with the keys
  float k8[E], k16[E];
  bool pr[E];
  int np = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {  // the keys' loads do not wait for the flags'
    const int j = lane + 32 * i;
    pr[i] = j < nb && (bf[j] & BF_KEY);
    k8[i] = j < nb ? e8[j] : 0.f;
    k16[i] = j < nb ? e16[j] : 0.f;
    np += pr[i] ? 1 : 0;
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) np += __shfl_xor_sync(0xffffffffu, np, m);
  const int r = min(min(th.rank_r, MAX_RANK_R), np);
  // the two top-r lists
  KI p8{INFINITY, -1}, p16{INFINITY, -1};
  for (int k = 0; k < r; ++k) {
    KI c8{-INFINITY, 0x7fffffff}, c16{-INFINITY, 0x7fffffff};
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if (!pr[i]) continue;
      const KI a{k8[i], lane + 32 * i}, a2{k16[i], lane + 32 * i};
      if (before(p8, a) && before(a, c8)) c8 = a;
      if (before(p16, a2) && before(a2, c16)) c16 = a2;
    }
    p8 = warp_best(c8);
    p16 = warp_best(c16);
    if (lane == 0) {
      top8[w][k] = p8.i;
      top16[w][k] = p16.i;
    }
  }
  __syncwarp();
  // union: the INT8 list, then the FP16 entries it does not hold
  int base = r;
  for (int k0 = 0; k0 < r; k0 += 32) {
    const int k = k0 + lane;
    bool fresh = false;
    if (k < r) {
      fresh = true;
      for (int i = 0; i < r; ++i) fresh &= top8[w][i] != top16[w][k];
    }
    const unsigned m = __ballot_sync(0xffffffffu, fresh);
    if (fresh) uni[w][base + __popc(m & ((1u << lane) - 1u))] = top16[w][k];
    base += __popc(m);
  }
  for (int k = lane; k < r; k += 32) uni[w][k] = top8[w][k];
  const int nu = base;
  __syncwarp();
  // the union's keys from the lanes that hold them (block a: lane a % 32, slot a / 32)
  for (int k0 = 0; k0 < nu; k0 += 32) {
    const int k = k0 + lane;
    const int a = k < nu ? uni[w][k] : 0;
    const int sl = a >> 5, src = a & 31;
    float v8 = 0.f, v16 = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float x8 = __shfl_sync(0xffffffffu, k8[i], src);
      const float x16 = __shfl_sync(0xffffffffu, k16[i], src);
      if (sl == i) {
        v8 = x8;
        v16 = x16;
      }
    }
    if (k < nu) {
      u8[w][k] = v8;
      u16[w][k] = v16;
    }
  }
  __syncwarp();
  // discordant pairs of U: the two orders place the pair the other way round
  int disc = 0;
  for (int pi = lane; pi < nu * nu; pi += 32) {
    const int i = pi / nu, j = pi - i * nu;
    if (i >= j) continue;
    const int a = uni[w][i], c = uni[w][j];
    const bool a8 = before(KI{u8[w][i], a}, KI{u8[w][j], c});
    const bool a16 = before(KI{u16[w][i], a}, KI{u16[w][j], c});
    disc += a8 != a16 ? 1 : 0;
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) disc += __shfl_xor_sync(0xffffffffu, disc, m);
  const bool fail = disc > th.rank_tol;
  const bool naive = th.naive != 0;
  // one 64-bit arrival per head: the low word counts the row's rung-3 heads,
  // the high word the heads done, so the last head learns both at once
  unsigned long long* cnt = reinterpret_cast<unsigned long long*>(sc.dcnt + 2 * b);
  int last = 0, n3 = 0;
  if (lane == 0) {
    uint8_t hf = hf0;
    if (!naive && fail) hf |= HF_RANKFAIL;
    sc.hflags[row] = hf;
    const bool is3 = !naive && (hf & (HF_KEYFAIL | HF_RANKFAIL));
    __threadfence();  // this head's flags are visible before its arrival
    const unsigned long long old = atomicAdd(cnt, (1ull << 32) + (is3 ? 1ull : 0ull));
    last = (int)(old >> 32) == sh.Hq - 1;
    n3 = (int)(old & 0xffffffffull) + (is3 ? 1 : 0);
  }
  if (!__shfl_sync(0xffffffffu, last, 0)) return;
  // the last head of the batch row: rung 3 per head, or rung 4 for the layer
  __threadfence();
  n3 = __shfl_sync(0xffffffffu, n3, 0);
  const bool layer = !naive && n3 >= need_dense;
  for (int hh = lane; hh < sh.Hq; hh += 32) {
    const size_t rw = (size_t)b * sh.Hq + hh;
    const uint8_t hf = __ldcg(&sc.hflags[rw]);
    const bool is3 = !naive && (hf & (HF_KEYFAIL | HF_RANKFAIL));
    sc.dense[rw] = layer ? 4 : (is3 ? 3 : 0);
  }
  if (lane == 0) *cnt = 0ull;
}

// The same decision for rows of more than 256 blocks: one CTA of DT threads per
// (batch row, query head).  The head's INT8 and FP16
// block log-masses and the block flags are staged in shared memory when they
// fit (else read in place).  The two top-r lists are built one rank at a time
// by CTA-wide arg-bests under the (key desc, index asc) orders; their union U
// (at most 2 * MAX_RANK_R blocks) is then compared pair by pair, one pair per
// thread per round.  The last CTA of a batch row to finish takes the
// whole-layer decision (rung 4).
constexpr int DT = 256;
constexpr int DW = DT / 32;

__global__ void __launch_bounds__(DT) decide_cta_kernel(DecodeShape sh, cqa_thresholds th,
                                                    int need_dense, Scratch sc, int staged) {
  pdl_begin();
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ KI red[2][DW];
  __shared__ int cnt[DW];
  __shared__ int top8[MAX_RANK_R], top16[MAX_RANK_R];
  __shared__ int uni[2 * MAX_RANK_R];
  __shared__ int nuni;
  __shared__ int flag;
  const int row_i = blockIdx.x;  // b * Hq + h
  const int b = row_i / sh.Hq, h = row_i - b * sh.Hq;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = b * sh.Hkv + h / sh.G;
  const size_t row = (size_t)row_i;
  int nb, r_unused;  // this batch row's sealed blocks
  row_blocks(sh, b, nb, r_unused);
  const uint8_t* bf_g = sc.bflags + (size_t)unit * sh.nbm;
  const float* e8_g = sc.ell8 + row * sh.nbm;
  const float* e16_g = sc.ell16 + row * sh.nbm;
  const float* e8 = e8_g;
  const float* e16 = e16_g;
  const uint8_t* bf = bf_g;
  if (staged) {
    float* s8 = reinterpret_cast<float*>(dsm);
    float* s16 = s8 + nb;
    uint8_t* sb = reinterpret_cast<uint8_t*>(s16 + nb);
    for (int j = tid; j < nb; j += DT) {
      s8[j] = e8_g[j];
      s16[j] = e16_g[j];
      sb[j] = bf_g[j];
    }
    e8 = s8;
    e16 = s16;
    bf = sb;
    __syncthreads();
  }
  // promoted-block count
  int np = 0;
  for (int j = tid; j < nb; j += DT) np += (bf[j] & BF_KEY) ? 1 : 0;
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) np += __shfl_xor_sync(0xffffffffu, np, m);
  if (lane == 0) cnt[warp] = np;
  __syncthreads();
  np = 0;
#pragma unroll
  for (int w = 0; w < DW; ++w) np += cnt[w];
  const int r = min(min(th.rank_r, MAX_RANK_R), np);
  // the two top-r lists
  KI p8{INFINITY, -1}, p16{INFINITY, -1};
  for (int k = 0; k < r; ++k) {
    KI c8{-INFINITY, 0x7fffffff}, c16{-INFINITY, 0x7fffffff};
    for (int j = tid; j < nb; j += DT) {
      if (!(bf[j] & BF_KEY)) continue;
      const KI a{e8[j], j}, a2{e16[j], j};
      if (before(p8, a) && before(a, c8)) c8 = a;
      if (before(p16, a2) && before(a2, c16)) c16 = a2;
    }
    c8 = warp_best(c8);
    c16 = warp_best(c16);
    __syncthreads();  // the previous round's reads of red are done
    if (lane == 0) {
      red[0][warp] = c8;
      red[1][warp] = c16;
    }
    __syncthreads();
    c8 = red[0][0];
    c16 = red[1][0];
#pragma unroll
    for (int w = 1; w < DW; ++w) {
      c8 = ki_best(c8, red[0][w]);
      c16 = ki_best(c16, red[1][w]);
    }
    p8 = c8;
    p16 = c16;
    if (tid == 0) {
      top8[k] = p8.i;
      top16[k] = p16.i;
    }
  }
  __syncthreads();
  // union: the INT8 list, then the FP16 entries it does not hold (warp 0)
  if (warp == 0) {
    int base = r;
    for (int k0 = 0; k0 < r; k0 += 32) {
      const int k = k0 + lane;
      bool fresh = false;
      if (k < r) {
        fresh = true;
        for (int i = 0; i < r; ++i) fresh &= top8[i] != top16[k];
      }
      const unsigned m = __ballot_sync(0xffffffffu, fresh);
      if (fresh) uni[base + __popc(m & ((1u << lane) - 1u))] = top16[k];
      base += __popc(m);
    }
    for (int k = lane; k < r; k += 32) uni[k] = top8[k];
    if (lane == 0) nuni = base;
  }
  __syncthreads();
  // discordant pairs of U: the two orders place the pair the other way round
  const int nu = nuni;
  int disc = 0;
  for (int pi = tid; pi < nu * nu; pi += DT) {
    const int i = pi / nu, j = pi - i * nu;
    if (i >= j) continue;
    const int a = uni[i], c = uni[j];
    const bool a8 = before(KI{e8[a], a}, KI{e8[c], c});
    const bool a16 = before(KI{e16[a], a}, KI{e16[c], c});
    disc += a8 != a16 ? 1 : 0;
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) disc += __shfl_xor_sync(0xffffffffu, disc, m);
  __syncthreads();  // cnt was read above
  if (lane == 0) cnt[warp] = disc;
  __syncthreads();
  disc = 0;
#pragma unroll
  for (int w = 0; w < DW; ++w) disc += cnt[w];
  const bool fail = disc > th.rank_tol;
  const bool naive = th.naive != 0;
  if (tid == 0) {
    uint8_t hf = sc.hflags[row];
    if (!naive && fail) hf |= HF_RANKFAIL;
    sc.hflags[row] = hf;
    const bool is3 = !naive && (hf & (HF_KEYFAIL | HF_RANKFAIL));
    if (is3) atomicAdd(&sc.dcnt[2 * b], 1);
    __threadfence();
    flag = atomicAdd(&sc.dcnt[2 * b + 1], 1) == sh.Hq - 1;
  }
  __syncthreads();
  if (!flag) return;
  // the last head of the batch row: rung 3 per head, or rung 4 for the layer
  __threadfence();
  const int n3 = atomicAdd(&sc.dcnt[2 * b], 0);
  const bool layer = !naive && n3 >= need_dense;
  for (int hh = tid; hh < sh.Hq; hh += DT) {
    const size_t rw = (size_t)b * sh.Hq + hh;
    const uint8_t hf = __ldcg(&sc.hflags[rw]);
    const bool is3 = !naive && (hf & (HF_KEYFAIL | HF_RANKFAIL));
    sc.dense[rw] = layer ? 4 : (is3 ? 3 : 0);
  }
  if (tid == 0) {
    sc.dcnt[2 * b] = 0;
    sc.dcnt[2 * b + 1] = 0;
  }
}

// Outputs, E_val and the E_val post-check; one CTA of MERGE_THREADS threads per
// (batch row, head).
template <int D, int G>
__global__ void __launch_bounds__(MERGE_THREADS)
    combine_kernel(DecodeShape sh, cqa_thresholds th, Scratch sc, float* __restrict__ out,
                   float* __restrict__ e_key, float* __restrict__ e_val,
                   uint8_t* __restrict__ rung) {
  pdl_begin();
  const int row = blockIdx.x;  // b * Hq + h
  const int b = row / sh.Hq, h = row - b * sh.Hq;
  const int g = h / G, hh = h - g * G;
  const size_t base = ((size_t)b * sh.Hkv + g) * sc.max_chunks * G + hh;
  const MergeStats ms = merge_parts<D, G>(sc, base, sh.nchunks, false, out + (size_t)row * D);
  if (threadIdx.x != 0) return;
  const uint8_t dv = sc.dense[row];
  uint8_t hf = sc.hflags[row];
  const float ev = ms.E / ms.L;
  if (dv) {
    e_key[row] = 0.f;
    e_val[row] = 0.f;
    rung[row] = dv;
  } else if (!th.naive && ev > th.eps_val) {
    // post-check failure: exact attention follows in a separate dense pass
    hf |= HF_VALFAIL;
    sc.dense[row] = 3 | DENSE_LATE;
    e_key[row] = 0.f;
    e_val[row] = 0.f;
    rung[row] = 3;
  } else {
    e_key[row] = sc.ekey[row];
    e_val[row] = ev;
    rung[row] = (hf & HF_VALUE) ? 2 : ((hf & HF_WIDENED) ? 1 : 0);
  }
  sc.hflags[row] = hf;
}

// One CTA of MERGE_THREADS threads per (batch row, query head): heads
// recomputed by a dense pass (all heads for cqa_dense_reference, DENSE_LATE
// heads otherwise).
template <int D, int G>
__global__ void __launch_bounds__(MERGE_THREADS)
    dense_combine_kernel(DecodeShape sh, Scratch sc, int all_heads, float* __restrict__ out,
                         float* __restrict__ e_key, float* __restrict__ e_val,
                         uint8_t* __restrict__ rung) {
  pdl_begin();
  const int row = blockIdx.x;  // b * Hq + h
  const int b = row / sh.Hq, h = row - b * sh.Hq;
  if (!all_heads && !(sc.dense[row] & DENSE_LATE)) return;
  const int g = h / G, hh = h - g * G;
  const size_t base = ((size_t)b * sh.Hkv + g) * sc.max_chunks * G + hh;
  merge_parts<D, G>(sc, base, sh.nchunks, false, out + (size_t)row * D);
  if (!all_heads && threadIdx.x == 0) {
    e_key[row] = 0.f;
    e_val[row] = 0.f;
    rung[row] = 3;
  }
}

template <int D, int G>
cudaError_t combine_t(const DecodeShape& sh, const cqa_thresholds& th, const Scratch& sc,
                      float* out, float* e_key, float* e_val, uint8_t* rung, cudaStream_t s) {
  return launch_pdl(combine_kernel<D, G>, dim3(sh.B * sh.Hq), dim3(MERGE_THREADS), 0, s, sh, th, sc, out, e_key,
                    e_val, rung);
}

template <int D, int G>
cudaError_t dense_combine_t(const DecodeShape& sh, const Scratch& sc, int all_heads, float* out,
                            float* e_key, float* e_val, uint8_t* rung, cudaStream_t s) {
  return launch_pdl(dense_combine_kernel<D, G>, dim3(sh.B * sh.Hq), dim3(MERGE_THREADS), 0, s, sh, sc,
                    all_heads, out, e_key, e_val, rung);
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

cudaError_t launch_combine(const DecodeShape& sh, const cqa_thresholds& th, const Scratch& sc,
                           float* out, float* e_key, float* e_val, uint8_t* rung,
                           cudaStream_t s) {
  CQA_DISPATCH_DG(combine_t, sh, th, sc, out, e_key, e_val, rung, s);
}

cudaError_t launch_decide(const DecodeShape& sh, const cqa_thresholds& th, int need_dense,
                          const Scratch& sc, cudaStream_t s) {
  const dim3 grid((sh.B * sh.Hq + DWH - 1) / DWH), block(32 * DWH);
  if (sh.nb_max <= 32)
    return launch_pdl(decide_kernel<1>, grid, block, 0, s, sh, th, need_dense, sc);
  if (sh.nb_max <= 64)
    return launch_pdl(decide_kernel<2>, grid, block, 0, s, sh, th, need_dense, sc);
  if (sh.nb_max <= 128)
    return launch_pdl(decide_kernel<4>, grid, block, 0, s, sh, th, need_dense, sc);
  if (sh.nb_max <= 256)
    return launch_pdl(decide_kernel<8>, grid, block, 0, s, sh, th, need_dense, sc);
  // longer rows: a CTA per head, the head's keys and flags staged in shared
  // memory up to 96 KiB
  const size_t bytes = (size_t)sh.nb_max * 9;
  const int staged = bytes <= 96u * 1024u ? 1 : 0;
  const int smem = staged ? (int)((bytes + 15) / 16 * 16) : 0;
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_dynamic_smem((const void*)decide_cta_kernel, smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(decide_cta_kernel, dim3(sh.B * sh.Hq), dim3(DT), smem, s, sh, th, need_dense,
                    sc, staged);
}

cudaError_t launch_dense_combine(const DecodeShape& sh, const Scratch& sc, int all_heads,
                                 float* out, float* e_key, float* e_val, uint8_t* rung,
                                 cudaStream_t s) {
  CQA_DISPATCH_DG(dense_combine_t, sh, sc, all_heads, out, e_key, e_val, rung, s);
}

}  // namespace cqa
