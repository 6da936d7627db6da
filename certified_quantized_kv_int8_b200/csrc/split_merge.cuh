// Merge of the split-K partials of one (batch row, query head), shared by the
// combine kernels of the certified pass, of the dense passes and of the
// INT8/INT4 streaming pass.
//
// Runtime-Certified Bounded-Error Quantized Attention, Methodology §2: the
// output is the softmax-weighted sum over all blocks, and E_val the attention
// mass of the INT4-valued blocks times their eta_b; split-K partials carry,
// per part, the running max m, the sum l of exp(x - m), the eta mass e (in the
// same scale as l) and the unnormalised output vector, so that
//   o = sum_c exp(m_c - M) o_c / L,  L = sum_c exp(m_c - M) l_c,
//   E = sum_c exp(m_c - M) e_c,      M = max_c m_c.
//
// One CTA of MERGE_THREADS threads.  The parts' output vectors are spread over
// the warps (a warp instruction covers 32 / (D / 4) parts), and each lane loads
// its first MERGE_PRE parts before the statistics are known, so those loads
// overlap the statistics' own.  Every warp then reduces the statistics over
// all parts by itself with shuffles, which needs no barrier; the one CTA
// barrier comes before the warps' vectors are summed in shared memory.
#pragma once

#include "cqa_internal.cuh"

namespace cqa {

constexpr int MERGE_THREADS = 512;  // sixteen warps
constexpr int MERGE_PRE = 5;        // parts per lane loaded ahead: five rounds of sixteen
                                    // warps cover 80 parts at head_dim 128

__device__ __forceinline__ float merge_warp_max(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ float merge_warp_sum(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

struct MergeStats {
  float M;   // largest part max
  float L;   // softmax denominator at M
  float E;   // eta mass at M
  float XA;  // largest part_x[0] over the parts (only when asked for)
};

// Parts 0 .. nparts-1 of the head whose part 0 has partial index `base`
// (part c: index base + c * G).  Writes o / L to out_row[0 .. D) and returns
// the statistics to every thread.  with_x: also reduce the max of
// part_x[3 * index] (the streaming pass's largest Delta).
template <int D, int G>
__device__ __forceinline__ MergeStats merge_parts(const Scratch& sc, size_t base, int nparts,
                                                  bool with_x, float* __restrict__ out_row) {
  constexpr int NWC = MERGE_THREADS / 32;
  constexpr int V4 = D / 4;          // float4 items of an output vector
  constexpr int PPW = 32 / V4;       // parts per warp instruction
  constexpr int SLOTS = NWC * PPW;   // parts in flight per round
  static_assert(PPW >= 1 && 32 % V4 == 0, "head_dim");
  __shared__ float4 red[SLOTS][V4];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* ps = sc.part_s + base * 3;  // part c: ps[c * G * 3 + {m, l, e}]
  const float* px = sc.part_x + base * 3;  // part c: px[c * G * 3]
  const float4* po = reinterpret_cast<const float4*>(sc.part_o + base * D);
  const int vi = lane % V4, sl = warp * PPW + lane / V4;

  float4 v[MERGE_PRE];
  float mv[MERGE_PRE];
#pragma unroll
  for (int i = 0; i < MERGE_PRE; ++i) {
    const int c = sl + i * SLOTS;
    const bool in = c < nparts;
    v[i] = in ? po[(size_t)c * G * V4 + vi] : make_float4(0.f, 0.f, 0.f, 0.f);
    mv[i] = in ? ps[(size_t)c * G * 3] : -INFINITY;
  }
  MergeStats st;
  float M = -INFINITY, xa = 0.f;
  for (int c = lane; c < nparts; c += 32) {
    M = fmaxf(M, ps[(size_t)c * G * 3]);
    if (with_x) xa = fmaxf(xa, px[(size_t)c * G * 3]);
  }
  M = merge_warp_max(M);
  st.XA = with_x ? merge_warp_max(xa) : 0.f;
  float ll = 0.f, el = 0.f;
  for (int c = lane; c < nparts; c += 32) {
    const float* p = ps + (size_t)c * G * 3;
    const float m = p[0];
    const float w = m == -INFINITY ? 0.f : expf(m - M);
    ll = fmaf(p[1], w, ll);
    el = fmaf(p[2], w, el);
  }
  st.M = M;
  st.L = merge_warp_sum(ll);
  st.E = merge_warp_sum(el);

  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < MERGE_PRE; ++i) {
    const float w = mv[i] == -INFINITY ? 0.f : expf(mv[i] - M);
    o.x = fmaf(v[i].x, w, o.x);
    o.y = fmaf(v[i].y, w, o.y);
    o.z = fmaf(v[i].z, w, o.z);
    o.w = fmaf(v[i].w, w, o.w);
  }
  for (int c = sl + MERGE_PRE * SLOTS; c < nparts; c += SLOTS) {  // beyond the first rounds
    const float m = ps[(size_t)c * G * 3];
    const float w = m == -INFINITY ? 0.f : expf(m - M);
    const float4 t = po[(size_t)c * G * V4 + vi];
    o.x = fmaf(t.x, w, o.x);
    o.y = fmaf(t.y, w, o.y);
    o.z = fmaf(t.z, w, o.z);
    o.w = fmaf(t.w, w, o.w);
  }
  red[sl][vi] = o;
  __syncthreads();
  const float il = 1.f / st.L;
  for (int i = tid; i < V4; i += MERGE_THREADS) {
    float4 s = red[0][i];
    for (int k = 1; k < SLOTS; ++k) {
      const float4 t = red[k][i];
      s.x += t.x;
      s.y += t.y;
      s.z += t.z;
      s.w += t.w;
    }
    reinterpret_cast<float4*>(out_row)[i] = make_float4(s.x * il, s.y * il, s.z * il, s.w * il);
  }
  return st;
}

}  // namespace cqa
