/*
 * cqa.h — C ABI of the certified quantized KV-cache decode-attention library
 * (libcqa.so, CUDA for sm_100a).
 *
 * The library implements the decode-step hot path of *Runtime-Certified
 * Bounded-Error Quantized Attention* (gist.science summary of paper
 * 2605.20868, technical summary):
 *   - Methodology §1 "Tiered storage with deterministic fallback": Tier 1 in
 *     device memory (per-channel INT8 keys, per-group INT4 values, their
 *     scales/offsets, per-block error annotations eta_b); Tier 2 in pinned
 *     host RAM (the FP16 originals).
 *   - Methodology §2 "Two-term error decomposition": per head and step, a key
 *     bound E_key (total-variation distance of the softmax, from the per-token
 *     score perturbation Delta) and a value bound E_val (attention mass times
 *     eta_b), computed from Tier-1 quantities only.
 *   - Methodology §3 "Adaptive precision and fallback ladder": an INT8 scoring
 *     pass, promotion of the top-K* blocks covering tau_cov of the estimated
 *     mass to FP16 keys paged from Tier 2, a block-ranking consistency check,
 *     and the four rungs (widen coverage, FP16 values, per-head dense,
 *     whole-layer dense).
 *
 * Conventions for every entry point:
 *   - Return value: CQA_OK (0) or a negative CQA_ERR_* code; cqa_error_string
 *     names it.  On an argument error nothing is launched and no output is
 *     written.  CQA_ERR_CUDA reports a failed CUDA call; the cache may then be
 *     in an unspecified state and should be destroyed.
 *   - Device pointers are plain CUDA device addresses (cudaMalloc or any
 *     allocator of the same device); `stream` is a cudaStream_t passed as
 *     void* (NULL = the legacy default stream).  Calls enqueue work on
 *     `stream` and return; results are valid once the stream has synchronised.
 *   - Ownership: the caller owns every pointer it passes; the library owns
 *     both tiers and all scratch memory held by a cqa_cache.
 *   - Threading: a cache may be used by one host thread at a time, and two
 *     calls on one cache must not overlap on the GPU (use one stream, or order
 *     the streams).
 *   - Layouts are row-major C arrays; "fp16" is IEEE binary16.
 */
#ifndef CQA_H
#define CQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  CQA_OK = 0,
  CQA_ERR_INVALID_ARG = -1, /* null pointer, bad shape, layer out of range, ... */
  CQA_ERR_CUDA = -2,        /* a CUDA runtime call failed */
  CQA_ERR_OOM = -3,         /* device or pinned-host allocation failed */
  CQA_ERR_CAPACITY = -4,    /* an append beyond max_ctx, or a shape beyond a fixed scratch size */
  CQA_ERR_EMPTY = -5,       /* decode on a layer that holds no token */
  CQA_ERR_TIMEOUT = -6      /* reported by cqa_device_status: a device wait gave up */
};

typedef struct cqa_cache cqa_cache; /* opaque */

/* Shape of one cache: every layer holds `batch` sequences.  Rows may hold
 * different lengths (ragged batch): cqa_quantize_append_row grows one row,
 * cqa_quantize_append grows every row by the same count. */
typedef struct cqa_config {
  int32_t n_layers;
  int32_t batch;
  int32_t n_q_heads;  /* query heads; query head h reads kv head h / (n_q_heads / n_kv_heads) */
  int32_t n_kv_heads; /* must divide n_q_heads; n_q_heads / n_kv_heads in {1, 2, 4, 8} */
  int32_t head_dim;   /* 64 or 128 */
  int32_t max_ctx;    /* token capacity per (layer, batch row), >= 1 */
  int32_t device;     /* CUDA device ordinal the cache lives on */
  int32_t meta_fp16;  /* Tier-1 metadata precision (Methodology §1 leaves it open):
                         0: key scales and value scale/offset in float32 (232 B per token
                         and kv head at head_dim 128); 1: in binary16 (212 B): each
                         scale is rounded up to binary16 before the codes are taken
                         against it, so no code clamps and the stored scale still bounds
                         the rounding error; the value offset (a group min of binary16
                         inputs) is stored exactly */
} cqa_config;

/* Largest rank_r a decode accepts (CQA_ERR_INVALID_ARG above it). */
#define CQA_MAX_RANK_R 64

/* Runtime thresholds of one decode call (Methodology §3).  tau_cov and v_tol
 * are named by the method; the other fields are this library's readings of
 * triggers the method leaves unstated. */
typedef struct cqa_thresholds {
  float tau_cov;          /* promote the fewest blocks whose INT8-estimated mass, plus the
                             exact residual block, reaches tau_cov; >= 1 promotes all */
  float eps_key;          /* rung 1: widen K* (doubling) while E_key > eps_key ... */
  int32_t max_expand;     /* ... at most max_expand times; still above -> rung 3 */
  float v_tol;            /* rung 2: FP16 values for block b if some head's
                             m8_b * eta_b > v_tol (m8 = INT8-estimated block mass) */
  int32_t rank_r;         /* rank check (Methodology §3, rank-consistency check): over the
                             promoted blocks, the top-min(rank_r, |P|) blocks by INT8 and by
                             FP16 block log-mass (ties to the lower block index) form a union
                             U; the rankings disagree when more than rank_tol pairs of U are
                             ordered the other way round by the two log-masses -> rung 3.
                             0 <= rank_r <= CQA_MAX_RANK_R; 0 disables the check */
  float eps_val;          /* rung 3 also when E_val > eps_val (+inf disables) */
  float layer_dense_frac; /* rung 4 when >= ceil(layer_dense_frac * n_q_heads) heads of a
                             (layer, batch row) took rung 3 by the rank check or by E_key */
  int32_t naive;          /* 1: certification off (no promotion, no ladder; bounds still
                             reported; one fused INT8/INT4 streaming pass), 0: certified */
  int32_t rank_tol;       /* discordant pairs of U the rank check tolerates (>= 0); 0 makes
                             it require equal ordered top-r lists */
} cqa_thresholds;

/* Optional per-call diagnostics, all device pointers, any may be NULL.
 * nb = number of sealed 64-token blocks of the layer's longest row
 * (length / 64); in a shorter row, entries past its own sealed blocks are
 * unspecified. */
typedef struct cqa_trace {
  int32_t* kstar;       /* [batch][n_q_heads] final K* after widening */
  uint8_t* block_flags; /* [batch][n_kv_heads][nb]: bit0 key promoted, bit1 value promoted */
  float* ell8;          /* [batch][n_q_heads][nb] INT8 block log-mass (natural log) */
  float* ell16;         /* [batch][n_q_heads][nb] FP16 block log-mass, promoted blocks only */
  float* delta;         /* [batch][n_q_heads][nb] per-token score perturbation bound Delta */
  uint8_t* head_flags;  /* [batch][n_q_heads]: bit0 widened, bit1 value promotion,
                           bit2 E_key fail, bit3 rank fail, bit4 E_val fail */
  float* ell_res;       /* [batch][n_q_heads] log-mass of the exact residual block (-inf if empty) */
} cqa_trace;

/* Allocate both tiers for `cfg` on cfg->device (Methodology §1, tiered
 * storage: Tier 1 holds the compressed cache in device memory, Tier 2 the FP16
 * originals in pinned system RAM): Tier 1 and scratch in device memory, Tier 2
 * (n_layers * batch * n_kv_heads * max_ctx * head_dim * 2 fp16) in pinned,
 * device-mapped host memory, and the two key-staging buffers of
 * cqa_set_key_prefetch.  *out receives the handle.  CQA_ERR_INVALID_ARG for an
 * unsupported shape, CQA_ERR_OOM when a device or pinned allocation fails
 * (everything allocated so far is freed and *out stays NULL). */
int cqa_cache_create(const cqa_config* cfg, cqa_cache** out);

/* Free everything the cache owns (synchronises the device first).  NULL is a no-op. */
int cqa_cache_destroy(cqa_cache* cache);

/* Tokens currently held by `layer`: the longest batch row's length
 * (host-side counter; no synchronisation). */
int cqa_cache_length(const cqa_cache* cache, int layer, int32_t* out_len);

/* Tokens held by each batch row of `layer`: out_lens is a host array of
 * `batch` int32 (host-side counters; no synchronisation). */
int cqa_cache_row_lengths(const cqa_cache* cache, int layer, int32_t* out_lens);

/* Append n_new tokens to every batch row of `layer` (Methodology §1), each
 * after its own row's tokens (rows of different lengths stay ragged).
 * k_fp16, v_fp16: device fp16 [batch][n_kv_heads][n_new][head_dim].
 * Every complete 64-token block is sealed: keys -> symmetric INT8 with one
 * fp32 scale per (block, channel) (s = amax/127, code = round-half-even(k/s)),
 * values -> asymmetric INT4 per (token, 32 channels) (z = min,
 * s = (max-min)/15), eta_b = max |v - (s*code + z)| over the block; the newest
 * length % 64 tokens stay exact in FP16 (the residual block, device memory).
 * A block's FP16 originals are written to Tier 2 when it seals (the residual
 * block is never promoted, so its tokens need no host copy before that).
 * The encoding of a block depends only on
 * its tokens, so appending in any chunking gives the same cache.
 * CQA_ERR_CAPACITY if length + n_new > max_ctx.  n_new = 0 is a no-op. */
int cqa_quantize_append(cqa_cache* cache, int layer, const void* k_fp16, const void* v_fp16,
                        int n_new, void* stream);

/* Append n_new tokens to batch row `row` of `layer` only, encoded exactly as
 * cqa_quantize_append encodes them; the other rows keep their lengths.
 * k_fp16, v_fp16: device fp16 [n_kv_heads][n_new][head_dim].
 * CQA_ERR_INVALID_ARG if row is outside [0, batch); CQA_ERR_CAPACITY if the
 * row's length + n_new > max_ctx.  n_new = 0 is a no-op. */
int cqa_quantize_append_row(cqa_cache* cache, int layer, int row, const void* k_fp16,
                            const void* v_fp16, int n_new, void* stream);

/* One certified decode step of `layer` for all batch rows (Methodology §2-§3),
 * each row over its own tokens (ragged rows allowed).
 * q_fp16: device fp16 [batch][n_q_heads][head_dim].
 * Outputs (device): out fp32 [batch][n_q_heads][head_dim]; e_key, e_val fp32
 * [batch][n_q_heads]; rung uint8 [batch][n_q_heads] = highest rung reached:
 * 0 certified as selected, 1 coverage widened, 2 FP16 values promoted,
 * 3 per-head dense, 4 whole-layer dense.  Dense heads return exact attention
 * over the FP16 originals with e_key = e_val = 0.  For the other heads
 * max_c |out - O_dense| <= R_V * e_key + e_val, R_V = max_c (vmax_c - vmin_c)
 * of the head's kv head (exported by cqa_debug_export).
 * th: host pointer.  trace: host pointer to a cqa_trace, or NULL.
 * CQA_ERR_EMPTY if some batch row of the layer holds no token. */
int cqa_decode(cqa_cache* cache, int layer, const void* q_fp16, const cqa_thresholds* th,
               float* out, float* e_key, float* e_val, uint8_t* rung, const cqa_trace* trace,
               void* stream);

/* Exact attention softmax(q K^T / sqrt(head_dim)) V of `layer` over the FP16
 * originals (Tier 2 plus the residual block), fp32 accumulation: the O_dense
 * that deterministic recovery returns (Key Contributions; Methodology §1,
 * fallback mechanism) and the dense rungs 3-4 of the ladder compute.  q_fp16 and out as in cqa_decode, each row
 * over its own tokens; CQA_ERR_EMPTY if some row holds no token. */
int cqa_dense_reference(cqa_cache* cache, int layer, const void* q_fp16, float* out, void* stream);

/* Copy one Tier-1 array of `layer` to host memory (synchronous; for tests and
 * inspection).  `what` selects the array, laid out as stated, with nb the
 * layer's sealed block count and d = head_dim.  In a ragged layer each
 * (batch row, kv head) takes its own row's extent (its nb, length % 64 and
 * length), and the units follow one another in [batch][n_kv_heads] order:
 *   CQA_EXPORT_KCODES   int8  [batch][n_kv_heads][nb][64][d]
 *   CQA_EXPORT_KSCALE   fp32  [batch][n_kv_heads][nb][d]  (binary16 metadata is
 *                       exported widened to fp32, exactly, like VMETA)
 *   CQA_EXPORT_VCODES   uint8 [batch][n_kv_heads][nb][64][d/2]  (channel 2j low nibble)
 *   CQA_EXPORT_VMETA    fp32  [batch][n_kv_heads][nb][64][d/32][2]  (scale, offset)
 *   CQA_EXPORT_ETA      fp32  [batch][n_kv_heads][nb]
 *   CQA_EXPORT_VRANGE   fp32  [batch][n_kv_heads][2][d]  (vmin, vmax over all tokens)
 *   CQA_EXPORT_RESIDUAL fp16  [batch][n_kv_heads][2][length % 64][d]  (keys, values)
 *   CQA_EXPORT_TIER2    fp16  [batch][n_kv_heads][2][length][d]  (keys, values: the
 *                       sealed tokens from Tier 2, the residual block's from device)
 * `bytes` must equal the array's size (CQA_ERR_INVALID_ARG otherwise);
 * cqa_debug_export(cache, layer, what, NULL, 0) returns that size instead
 * (as a non-negative value, or a negative error). */
enum {
  CQA_EXPORT_KCODES = 0,
  CQA_EXPORT_KSCALE = 1,
  CQA_EXPORT_VCODES = 2,
  CQA_EXPORT_VMETA = 3,
  CQA_EXPORT_ETA = 4,
  CQA_EXPORT_VRANGE = 5,
  CQA_EXPORT_RESIDUAL = 6,
  CQA_EXPORT_TIER2 = 7
};
int64_t cqa_debug_export(cqa_cache* cache, int layer, int what, void* host_dst, size_t bytes);

/* Device status word of the cache's kernels, read after synchronising the
 * device and then cleared.  The streaming kernels wait for their own bulk
 * copies with a bounded number of polls; a wait that runs out sets bit 0
 * (and that kernel's results are not valid).
 * *status = 0 means every kernel since the last call completed normally.  A
 * nonzero status also resets the kernels' arrival counters. */
int cqa_device_status(cqa_cache* cache, int32_t* status);

/* Self-test of the failure path above: launches one kernel that waits, for at
 * most `polls` polls, on a barrier nobody completes.  The wait gives up and
 * sets bit 0 of the status word, which the next cqa_device_status returns;
 * nothing faults or hangs.  Runs on the legacy default stream. */
int cqa_selftest_bounded_wait(cqa_cache* cache, int32_t polls);

/* Host-side fault injection, a test hook for the library's error paths
 * (Key Contributions: recovery must be deterministic, so its failure paths are
 * exercised without faulting a GPU).  Off unless armed; process-wide.  The
 * armed site fails once, on the host and without calling CUDA for it, after
 * `skip` of its calls have passed, and then disarms:
 *   CQA_FAULT_PINNED_ALLOC  a pinned host allocation of cqa_cache_create (there
 *                           are three: Tier-2 keys, Tier-2 values, the promotion
 *                           counters); the create returns CQA_ERR_OOM after
 *                           freeing everything it had allocated;
 *   CQA_FAULT_PREFETCH_COPY a copy of the whole-layer key prefetch; cqa_decode
 *                           returns CQA_ERR_CUDA before launching any kernel, so
 *                           its outputs are left untouched, and the slot is
 *                           marked empty.
 * CQA_FAULT_NONE disarms.  CQA_ERR_INVALID_ARG for an unknown site or skip < 0.
 * Arming is not synchronised with calls made by other threads. */
enum { CQA_FAULT_NONE = 0, CQA_FAULT_PINNED_ALLOC = 1, CQA_FAULT_PREFETCH_COPY = 2 };
int cqa_test_inject_fault(int site, int skip);

/* Whole-layer key prefetch.  Promotion reads the FP16 keys of the selected
 * blocks from Tier 2.  When a layer's last decode promoted nearly all of its
 * blocks, copying the layer's sealed keys to device memory with the copy
 * engine is faster than gathering them block by block, and the copy of the
 * next layer can run while the current layer computes.  With mode 1
 * (adaptive, the default) cqa_decode of layer l stages layer l (unless already
 * staged) and layer (l + 1) % n_layers whenever their last decode promoted at
 * least min_fraction of their blocks (the first decode of a layer never does);
 * mode 2 always stages; mode 0 never does.  Staging changes no result: the
 * promoted keys are the same bytes, and blocks the copy did not cover are
 * read from Tier 2 as before.  It uses two device buffers of one layer's
 * keys each (batch * n_kv_heads * max_ctx * head_dim fp16), allocated by
 * cqa_cache_create, and a copy stream owned by the cache. */
int cqa_set_key_prefetch(cqa_cache* cache, int mode, float min_fraction);

/* Per-phase device time of the library's kernels (tracing).  Between
 * cqa_profile_begin and cqa_profile_end, every kernel the cache launches is
 * bracketed by two CUDA events recorded on the call's stream; end waits for
 * them and reports, per phase, the summed event time in milliseconds and the
 * number of kernel launches.  Phases: */
enum {
  CQA_PHASE_APPEND_SEAL = 0,   /* sealing complete blocks into Tier 1 and Tier 2 */
  CQA_PHASE_APPEND_TAIL = 1,   /* residual block, value ranges */
  CQA_PHASE_SCORE = 2,         /* INT8 scoring pass */
  CQA_PHASE_SELECT = 3,        /* coverage selection, E_key, rungs 1-2 */
  CQA_PHASE_PROMOTE = 4,       /* FP16 keys of promoted blocks from Tier 2: exact logits */
  CQA_PHASE_DECIDE = 5,        /* rank check, rungs 3-4 */
  CQA_PHASE_DENSE_KEYS = 6,    /* exact logits of not-promoted blocks for dense heads */
  CQA_PHASE_ATTEND = 7,        /* split-K softmax and P.V, value bound */
  CQA_PHASE_COMBINE = 8,       /* split-K combine, E_val */
  CQA_PHASE_DENSE_ATTEND = 9,  /* exact attention from Tier 2 (E_val post-check, reference) */
  CQA_PHASE_DENSE_COMBINE = 10,
  CQA_PHASE_PREFETCH = 11,     /* copy-engine copy of a layer's Tier-2 keys (not a kernel) */
  CQA_PHASE_NAIVE = 12,        /* certification off: one streaming pass over Tier 1 */
  CQA_PHASE_NAIVE_COMBINE = 13, /* certification off: split-K combine, outputs and bounds */
  CQA_PHASE_PROMOTE_STAGED = 14, /* count only, never timed: the CQA_PHASE_PROMOTE launches
                                  * that read the keys from a device copy staged by the
                                  * prefetch instead of from Tier 2 over the host link */
  CQA_PHASE_COUNT = 15
};
/* Start (or restart) profiling; max_launches bounds the recorded launches
 * (further launches are counted but not timed). */
int cqa_profile_begin(cqa_cache* cache, int max_launches);
/* Stop profiling.  ms[CQA_PHASE_COUNT] and launches[CQA_PHASE_COUNT] are host
 * arrays (either may be NULL).  Returns the number of launches left untimed
 * (>= 0) or a negative error. */
int cqa_profile_end(cqa_cache* cache, double* ms, int64_t* launches);

/* Size in bytes of the fixed device scratch array that
 * cqa_dense_attention_noalloc uses (every device that loads the library holds
 * one such array until the process exits). */
#define CQA_NOALLOC_SCRATCH_BYTES (4u << 20)

/* Exact attention softmax(q K^T / sqrt(head_dim)) V over FP16 keys and values
 * that the caller holds in device memory, computed without allocating any
 * memory.  The paper has no counterpart of this entry point.  It exists for
 * callers that cannot call cudaMalloc: hosts whose single device allocator is
 * owned by another framework under a fixed memory budget (a library that
 * allocates on its own there takes memory the host has already promised
 * elsewhere), and latency-critical paths where cudaMalloc/cudaFree may
 * synchronise the device and stall every stream.
 *
 * q_fp16: device fp16 [batch][n_q_heads][head_dim]; k_fp16, v_fp16: device
 * fp16 [batch][n_kv_heads][n_tokens][head_dim]; out: device fp32
 * [batch][n_q_heads][head_dim]; all 16-byte aligned, owned by the caller.
 * Supported shapes: head_dim 64 or 128; n_q_heads / n_kv_heads (an integer)
 * in {1, 2, 4, 8}, except 8 at head_dim 64; batch, heads and n_tokens >= 1;
 * batch * n_kv_heads <= 65535.  Other shapes return CQA_ERR_INVALID_ARG.
 * The split-K partials live in a file-scope device array of
 * CQA_NOALLOC_SCRATCH_BYTES; shapes whose partials cannot fit (batch *
 * n_kv_heads * (n_q_heads / n_kv_heads) * (head_dim + 3) * 4 bytes above it)
 * are rejected with CQA_ERR_CAPACITY before anything is launched.  The call
 * allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *
 * The first call on a device (the current device) looks up the array's device
 * address with cudaGetSymbolAddress; make that first call before any stream
 * capture.  Every call on a device shares the one array, which keeps the last
 * call's contents (each call rewrites every partial before reading it, so
 * nothing needs clearing); calls that overlap on the GPU race on it, so
 * serialise them (one stream, or streams ordered by events). */
int cqa_dense_attention_noalloc(const void* q_fp16, const void* k_fp16, const void* v_fp16,
                                int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                int n_tokens, float* out, void* stream);

/* Static description of an error code. */
const char* cqa_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* CQA_H */
