// Internal declarations shared by the CUDA sources of libcqa.so.
//
// Data layout in device memory (Tier 1) for one unit u = (layer, batch row,
// kv head), nbm = max_ctx / 64 block slots, d = head_dim:
//   kcodes int8  [nbm][64][d]        token-major: one 16-byte load = 16 channels
//   kscale fp32  [nbm][d]            per (block, channel) key scale
//   vcodes uint8 [nbm][64][d/2]      INT4 pairs, channel 2j in the low nibble
//   vmeta  fp32  [nbm][64][d/32][2]  per (token, group): scale, offset
//   (kscale and vmeta are binary16 instead when the cache stores its
//   metadata in half precision: Tier1::meta16)
//   eta    fp32  [nbm]               per-block max INT4 reconstruction error
//   vrange fp32  [2][d]              running per-channel value min and max
//   kres, vres fp16 [64][d]          the residual (unsealed) block, exact
// Tier 2 (pinned host, device-mapped): k2, v2 fp16 [max_ctx][d] per unit.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "cqa.h"

namespace cqa {

constexpr int BLK = 64;  // tokens per block
constexpr int VG = 32;   // channels per INT4 value group
constexpr int MAX_RANK_R = CQA_MAX_RANK_R;  // longest top-r list of the rank check

// bits of the per-block flag byte
constexpr uint8_t BF_KEY = 1;  // FP16 keys promoted
constexpr uint8_t BF_VAL = 2;  // FP16 values promoted
// bits of the per-head flag byte
constexpr uint8_t HF_WIDENED = 1;
constexpr uint8_t HF_VALUE = 2;
constexpr uint8_t HF_KEYFAIL = 4;
constexpr uint8_t HF_RANKFAIL = 8;
constexpr uint8_t HF_VALFAIL = 16;
// dense-flag byte: 3 or 4 = rung decided before the attention pass (its exact
// logits and FP16 values are used there); DENSE_LATE marks an E_val post-check
// failure that a separate dense pass recomputes
constexpr uint8_t DENSE_LATE = 0x80;

struct Tier1 {
  int8_t* kcodes;
  float* kscale;     // float32 metadata (meta16 = 0)
  uint8_t* vcodes;
  float* vmeta;
  __half* kscale_h;  // the same arrays as binary16 (meta16 = 1)
  __half* vmeta_h;
  int meta16;        // 1: key scales and value scale/offset stored as binary16
  float* eta;
  float* vrange;
  __half* kres;
  __half* vres;
  __half* k2;  // device view of Tier 2 keys
  __half* v2;  // device view of Tier 2 values
};

// element strides per unit
struct Strides {
  size_t kcodes, kscale, vcodes, vmeta, eta, vrange, res, tier2;
};

inline Strides make_strides(int nbm, int d, int max_ctx) {
  Strides s;
  s.kcodes = (size_t)nbm * BLK * d;
  s.kscale = (size_t)nbm * d;
  s.vcodes = (size_t)nbm * BLK * d / 2;
  s.vmeta = (size_t)nbm * BLK * (d / VG) * 2;
  s.eta = (size_t)nbm;
  s.vrange = (size_t)2 * d;
  s.res = (size_t)BLK * d;
  s.tier2 = (size_t)max_ctx * d;
  return s;
}

// Scratch of one decode call (device), sized for nbm blocks.
struct Scratch {
  float* logits;     // [B][Hq][ls]  INT8 logits (sealed) + exact residual logits
  float* ell8;       // [B][Hq][nbm]
  float* delta;      // [B][Hq][nbm]
  float* ell16;      // [B][Hq][nbm]
  float* ell_res;    // [B][Hq]
  float* ekey;       // [B][Hq]
  int32_t* kstar;    // [B][Hq]
  uint8_t* hflags;   // [B][Hq]
  uint8_t* bflags;   // [B][Hkv][nbm]
  uint8_t* dense;    // [B][Hq] 0, 3 or 4
  float* part_o;     // [B*Hkv][max_chunks][G][d]
  float* part_s;     // [B*Hkv][max_chunks][G][3]  (m, l, eta mass)
  int32_t* promo;    // [n_layers * B * Hkv] promoted block count per unit (pinned host, mapped)
  int* err;          // device error word (bit 0: a bounded wait gave up)
  float* part_x;     // [B*Hkv][max_chunks][G][3]  naive pass: (max Delta, residual m, residual l)
  int* dcnt;         // [B][2] rank check: rung-3 heads, heads done (0 between calls;
                     // 8-byte aligned: one 64-bit word per row)
  size_t ls;         // logits row stride = nbm * 64 + 64
  int max_chunks;
};

// Shape of one decode call.  Batch rows may hold different lengths: grids are
// sized for the longest row (nb_max sealed blocks) and every CTA reads the
// length of its own row from `lens`.
struct DecodeShape {
  int B, Hq, Hkv, G, d, nb_max, nbm, nchunks, chunk_blocks;
  long long items_sum;  // sum over (row, kv head) units of their work items
  int sms;              // streaming multiprocessors of the cache's device (grid sizing)
  const int32_t* lens;  // device [B]: tokens held by each batch row of the layer
  const int32_t* lens_host;  // the same lengths in host memory (grid sizing by launchers)
  float sigma;
};

// Sealed blocks and residual tokens of batch row b.
__device__ __forceinline__ void row_blocks(const DecodeShape& sh, int b, int& nb, int& r) {
  const int T = __ldg(sh.lens + b);
  nb = T / BLK;
  r = T - nb * BLK;
}

// Work items of a row in the streaming passes: its sealed blocks, then the
// residual block, which costs about two sealed ones when it holds tokens.
__host__ __device__ __forceinline__ int row_items(int nb, int r) { return nb + (r > 0 ? 2 : 1); }

// CTAs per (row, kv head) unit of a streaming pass whose grid targets `target`
// resident CTAs: units receive CTAs in proportion to their work items, so the
// rows of a ragged batch finish together; at most `cap`, at least one.  The
// host sizes the grid with the same integer arithmetic.
__host__ __device__ __forceinline__ int unit_ctas(int target, int items, long long items_sum,
                                                  int cap) {
  long long n = (long long)target * items / (items_sum > 0 ? items_sum : 1);
  if (n > cap) n = cap;
  return n < 1 ? 1 : (int)n;
}

// Programmatic dependent launch.  The kernels of a decode step are launched
// with programmatic stream serialization: a kernel's CTAs may be scheduled
// while the previous kernel on the stream drains.  Each such kernel first lets
// its own dependent be scheduled (once all of its CTAs have started), then
// waits until the previous kernel has completed and its writes are visible,
// before touching global memory, so only the launch and scheduling latency
// overlap, never a data dependence.
__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device) and
// again only when a launch needs more than already granted: the attribute
// call may stall the host, so it stays off the per-launch path.
cudaError_t ensure_dynamic_smem(const void* kernel, int bytes);

// ---- launchers (each returns the launch error, cudaSuccess on success) ----
cudaError_t launch_seal(const Tier1& t, const Strides& st, int layer_unit0, int B, int Hkv, int d,
                        const __half* knew, const __half* vnew, int T_old, int n_new, int nb_old,
                        int nb_new, cudaStream_t s);
// also stores T_old + n_new as the length of each of the B rows (lens_rows[0..B))
cudaError_t launch_append_tail(const Tier1& t, const Strides& st, int layer_unit0, int B, int Hkv,
                               int d, const __half* knew, const __half* vnew, int T_old,
                               int n_new, int nb_new, int32_t* lens_rows, cudaStream_t s);
cudaError_t launch_score(const Tier1& t, const Strides& st, int layer_unit0, const DecodeShape& sh,
                         const __half* q, const Scratch& sc, cudaStream_t s);
// mode 0: promoted blocks (exact logits in place, ell16); 1: the other blocks
// of units holding a dense head (exact logits of the dense heads).  Keys of
// blocks j < stage_nb are read from `kstage` (a device copy of the layer's
// Tier-2 keys, same per-unit layout), the others from Tier 2.
cudaError_t launch_promote(const Tier1& t, const Strides& st, int layer_unit0,
                           const DecodeShape& sh, const __half* q, const Scratch& sc, int mode,
                           const __half* kstage, int stage_nb, cudaStream_t s);
cudaError_t launch_decide(const DecodeShape& sh, const cqa_thresholds& th, int need_dense,
                          const Scratch& sc, cudaStream_t s);
cudaError_t launch_select(const Tier1& t, const Strides& st, int layer_unit0,
                          const DecodeShape& sh, const cqa_thresholds& th, const Scratch& sc,
                          cudaStream_t s);
// mode 0: certified (logits from scratch; block and dense flags choose the
// values), 1: dense from Tier 2 for heads flagged DENSE_LATE, 2: dense for all
cudaError_t launch_attend(const Tier1& t, const Strides& st, int layer_unit0,
                          const DecodeShape& sh, const __half* q, const Scratch& sc, int mode,
                          cudaStream_t s);
// certification off: one streaming pass over Tier 1 into split-K partials;
// with `trace` set the pass also writes the per-block ell8, Delta and block
// flags of the trace
cudaError_t launch_naive(const Tier1& t, const Strides& st, int layer_unit0, const DecodeShape& sh,
                         const __half* q, const Scratch& sc, float* out, float* e_key,
                         float* e_val, uint8_t* rung, int trace, cudaStream_t s);
// the combine of that pass's split-K partials into the outputs, E_key, E_val
cudaError_t launch_naive_combine(const DecodeShape& sh, const Scratch& sc, float* out,
                                 float* e_key, float* e_val, uint8_t* rung, cudaStream_t s);
cudaError_t launch_combine(const DecodeShape& sh, const cqa_thresholds& th, const Scratch& sc,
                           float* out, float* e_key, float* e_val, uint8_t* rung,
                           cudaStream_t s);
cudaError_t launch_dense_combine(const DecodeShape& sh, const Scratch& sc, int all_heads,
                                 float* out, float* e_key, float* e_val, uint8_t* rung,
                                 cudaStream_t s);

}  // namespace cqa
