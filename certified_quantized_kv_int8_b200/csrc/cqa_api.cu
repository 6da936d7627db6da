// C ABI of libcqa.so: cache management, argument checks, launch sequences.
// The declarations and their contracts are in include/cqa.h.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <map>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include "bulk_pipe.cuh"
#include "cqa_internal.cuh"

namespace cqa {
size_t select_smem_bytes(int G, int nb);

}

using namespace cqa;

namespace cqa {
cudaError_t ensure_dynamic_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> granted;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  int& g = granted[std::make_pair(kernel, dev)];
  if (bytes <= g) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) g = bytes;
  return e;
}
}  // namespace cqa

struct cqa_cache {
  cqa_config cfg;
  int G, nbm;
  int sms;             // streaming multiprocessors of the device
  Strides st;
  Tier1 t;
  Scratch sc;
  int32_t* len;        // host [n_layers][batch]: tokens of each batch row
  int32_t* lens_dev;   // device copy of len, written by the append kernels in stream order
  uint32_t* seal_gen;  // host [n_layers]: count of appends that sealed a block in the layer
  void* k2_host;
  void* v2_host;
  size_t tier2_bytes;  // per tier-2 array
  void* dev_block;     // one device allocation holding Tier 1 and scratch
  // profiling (cqa_profile_begin / cqa_profile_end)
  bool prof_on;
  std::vector<cudaEvent_t>* prof_events;
  std::vector<int>* prof_phase;
  size_t prof_max;
  int64_t prof_launches[CQA_PHASE_COUNT];
  int64_t prof_untimed;
  // whole-layer key prefetch by the copy engine (cqa_set_key_prefetch)
  int pref_mode;       // 0 off, 1 adaptive, 2 always
  float pref_min_frac; // adaptive: the layer's last decode promoted at least this fraction
  cudaStream_t side;   // copy stream
  __half* kstage[2];   // [B*Hkv][max_ctx][d] device copies of one layer's Tier-2 keys
  int stage_layer[2];  // layer held by each slot, -1 none
  int stage_nb[2];     // sealed blocks copied into the slot (of the layer's longest row)
  uint32_t stage_gen[2];  // seal_gen of the layer when the slot was filled
  cudaEvent_t ev_ready[2], ev_free[2], ev_main;
  int32_t* promo_host; // [n_layers * B * Hkv] promoted blocks of the last decode (mapped)
  int32_t* promo_dev;
};

namespace {

// Host-side fault injection (cqa_test_inject_fault): the armed site fails once,
// after `skip` calls of it have passed.  Off unless a caller arms it.
std::atomic<int> g_fault_site{CQA_FAULT_NONE};
std::atomic<int> g_fault_skip{0};

bool fault_hit(int site) {
  if (g_fault_site.load() != site) return false;
  if (g_fault_skip.fetch_sub(1) > 0) return false;
  g_fault_site.store(CQA_FAULT_NONE);
  return true;
}

// cudaHostAlloc, or the injected failure of a pinned allocation
cudaError_t pinned_alloc(void** p, size_t bytes, unsigned flags) {
  if (fault_hit(CQA_FAULT_PINNED_ALLOC)) {
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  return cudaHostAlloc(p, bytes, flags);
}

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess) ok = true;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Grid target of the attention and promotion passes.  Their registers allow two
// CTAs of 256 threads per SM.  Up to 8192 blocks of work (units x blocks) the
// passes are latency-bound and one wave of two CTAs per SM is fastest (32K
// context, one layer: 142 -> 136 us); above it, where the host-link reads of
// dense heads and unstaged keys want many loads in flight, four per SM (two
// waves) are (64K x B4: 1394 -> 1465 us with two).
int target_ctas(int sms, long long work) { return sms * (work <= 8192 ? 2 : 4); }

void chunking(int units, int nb, int sms, int* chunk_blocks, int* nchunks) {
  int per_unit = (target_ctas(sms, (long long)units * nb) + units - 1) / units;
  if (per_unit < 1) per_unit = 1;
  int cb = nb > 0 ? (nb + per_unit - 1) / per_unit : 1;
  if (cb < 1) cb = 1;
  *chunk_blocks = cb;
  int nc = nb > 0 ? (nb + cb - 1) / cb : 1;
  *nchunks = nc < 1 ? 1 : nc;
}

// Partial slots per unit: the most CTAs one unit may receive from the widest
// grid, the streaming pass's four per SM (a whole grid's worth split over one
// row's kv heads, when the other rows of a ragged batch are short), plus the
// residual block's slot.
int max_chunks_for(int Hkv, int sms) { return sms * 4 / Hkv + 2; }

const int32_t* row_lens(const cqa_cache* c, int layer) {
  return c->len + (size_t)layer * c->cfg.batch;
}

int max_len(const cqa_cache* c, int layer) {
  const int32_t* L = row_lens(c, layer);
  int m = 0;
  for (int b = 0; b < c->cfg.batch; ++b) m = L[b] > m ? L[b] : m;
  return m;
}

int min_len(const cqa_cache* c, int layer) {
  const int32_t* L = row_lens(c, layer);
  int m = L[0];
  for (int b = 1; b < c->cfg.batch; ++b) m = L[b] < m ? L[b] : m;
  return m;
}

// Grids cover the longest row; each CTA reads its own row's length on the device.
DecodeShape shape_of(const cqa_cache* c, int layer) {
  DecodeShape sh;
  sh.B = c->cfg.batch;
  sh.Hq = c->cfg.n_q_heads;
  sh.Hkv = c->cfg.n_kv_heads;
  sh.G = c->G;
  sh.d = c->cfg.head_dim;
  sh.nb_max = 0;
  sh.items_sum = 0;
  const int32_t* L = row_lens(c, layer);
  for (int b = 0; b < sh.B; ++b) {
    const int nb = L[b] / BLK, r = L[b] - (L[b] / BLK) * BLK;
    if (nb > sh.nb_max) sh.nb_max = nb;
    sh.items_sum += (long long)sh.Hkv * row_items(nb, r);
  }
  sh.nbm = c->nbm;
  sh.lens = c->lens_dev + (size_t)layer * sh.B;
  sh.lens_host = L;
  sh.sigma = (float)(1.0 / sqrt((double)sh.d));
  sh.sms = c->sms;
  chunking(sh.B * sh.Hkv, sh.nb_max, sh.sms, &sh.chunk_blocks, &sh.nchunks);
  return sh;
}

// A barrier nobody arrives on, waited for with a bounded number of polls: the
// wait must give up and record ERR_TIMEOUT instead of hanging.
__global__ void bounded_wait_selftest_kernel(int* err, uint32_t polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_init_fence();
  }
  __syncthreads();
  mbar_wait(&bar, 0, err, polls);
}

__global__ void fill_range_kernel(float* vr, size_t units, int d) {
  const size_t n = units * 2 * (size_t)d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % (2 * (size_t)d));
    vr[i] = c < d ? INFINITY : -INFINITY;
  }
}

// Run one launcher; when profiling, bracket it with events on `s`.
template <class F>
cudaError_t run_phase(cqa_cache* c, int phase, cudaStream_t s, int nlaunch, F&& fn) {
  if (!c->prof_on || nlaunch == 0) return fn();
  const size_t k = c->prof_phase->size();
  const bool timed = k < c->prof_max;
  if (timed) {
    while (c->prof_events->size() < 2 * (k + 1)) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return cudaErrorMemoryAllocation;
      c->prof_events->push_back(e);
    }
    cudaEventRecord((*c->prof_events)[2 * k], s);
  }
  const cudaError_t e = fn();
  if (timed) {
    cudaEventRecord((*c->prof_events)[2 * k + 1], s);
    c->prof_phase->push_back(phase);
  } else {
    c->prof_untimed += nlaunch;
  }
  c->prof_launches[phase] += nlaunch;
  return e;
}

// Fraction of the layer's sealed blocks its last decode promoted (-1 unknown).
double last_promoted_fraction(const cqa_cache* c, int layer) {
  const int Hkv = c->cfg.n_kv_heads;
  const size_t units = (size_t)c->cfg.batch * Hkv;
  const volatile int32_t* p = c->promo_host + (size_t)layer * units;
  const int32_t* L = row_lens(c, layer);
  long long n = 0, total = 0;
  for (size_t i = 0; i < units; ++i) {
    const int32_t v = p[i];
    if (v < 0) return -1.0;
    n += v;
    total += L[i / Hkv] / BLK;
  }
  return total > 0 ? (double)n / (double)total : -1.0;
}

bool want_prefetch(const cqa_cache* c, int layer) {
  if (c->pref_mode == 0) return false;
  if (max_len(c, layer) / BLK == 0) return false;
  if (c->pref_mode == 2) return true;
  return last_promoted_fraction(c, layer) >= c->pref_min_frac;
}

// The slot holding `layer`'s keys as they are now (no block sealed since), or -1.
int staged_slot(const cqa_cache* c, int layer) {
  for (int i = 0; i < 2; ++i)
    if (c->stage_layer[i] == layer && c->stage_gen[i] == c->seal_gen[layer]) return i;
  return -1;
}

// Copy the sealed blocks of `layer`'s Tier-2 keys into a device slot on the
// copy stream, after all work already queued on `s` (the appends that wrote
// them) and after the slot's last reader.  Each batch row copies its own
// sealed blocks (one copy for all rows when their block counts agree).
// Returns the slot, -1 when there is nothing to copy, or -2 when a CUDA call
// failed (the slot is then marked empty).
int issue_prefetch(cqa_cache* c, int layer, int avoid_slot, cudaStream_t s) {
  const int nb = max_len(c, layer) / BLK;
  if (nb == 0) return -1;
  int slot = staged_slot(c, layer);
  if (slot >= 0) return slot;
  slot = (avoid_slot == 0) ? 1 : 0;
  const int B = c->cfg.batch, Hkv = c->cfg.n_kv_heads;
  const size_t units = (size_t)B * Hkv;
  const size_t pitch = c->st.tier2 * 2;
  const size_t blk_bytes = (size_t)BLK * c->cfg.head_dim * 2;
  const char* src = (const char*)c->k2_host + (size_t)layer * units * pitch;
  const int32_t* L = row_lens(c, layer);
  bool same = true;
  for (int b = 1; b < B; ++b) same = same && (L[b] / BLK == L[0] / BLK);
  if (cudaEventRecord(c->ev_main, s) != cudaSuccess) return -2;
  if (cudaStreamWaitEvent(c->side, c->ev_main, 0) != cudaSuccess) return -2;
  if (cudaStreamWaitEvent(c->side, c->ev_free[slot], 0) != cudaSuccess) return -2;
  const int timed = c->prof_on ? 1 : 0;
  cudaError_t e = run_phase(c, CQA_PHASE_PREFETCH, c->side, timed, [&] {
    if (fault_hit(CQA_FAULT_PREFETCH_COPY)) return cudaErrorInvalidValue;
    if (same)
      return cudaMemcpy2DAsync(c->kstage[slot], pitch, src, pitch, (size_t)nb * blk_bytes, units,
                               cudaMemcpyHostToDevice, c->side);
    for (int b = 0; b < B; ++b) {
      const int nbr = L[b] / BLK;
      if (nbr == 0) continue;
      const size_t off = (size_t)b * Hkv * pitch;
      const cudaError_t e2 =
          cudaMemcpy2DAsync((char*)c->kstage[slot] + off, pitch, src + off, pitch,
                            (size_t)nbr * blk_bytes, Hkv, cudaMemcpyHostToDevice, c->side);
      if (e2 != cudaSuccess) return e2;
    }
    return cudaSuccess;
  });
  if (e != cudaSuccess || cudaEventRecord(c->ev_ready[slot], c->side) != cudaSuccess) {
    c->stage_layer[slot] = -1;
    return -2;
  }
  c->stage_layer[slot] = layer;
  c->stage_nb[slot] = nb;
  c->stage_gen[slot] = c->seal_gen[layer];
  return slot;
}

}  // namespace

extern "C" {

const char* cqa_error_string(int code) {
  switch (code) {
    case CQA_OK: return "ok";
    case CQA_ERR_INVALID_ARG: return "invalid argument";
    case CQA_ERR_CUDA: return "CUDA runtime error";
    case CQA_ERR_OOM: return "out of memory";
    case CQA_ERR_CAPACITY: return "size exceeds a fixed capacity (cache max_ctx or scratch size)";
    case CQA_ERR_EMPTY: return "decode on an empty layer";
    case CQA_ERR_TIMEOUT: return "a bounded device wait gave up (see cqa_device_status)";
  }
  return "unknown error";
}

int cqa_cache_create(const cqa_config* cfg, cqa_cache** out) {
  if (!cfg || !out) return CQA_ERR_INVALID_ARG;
  *out = nullptr;
  const cqa_config c = *cfg;
  if (c.n_layers < 1 || c.batch < 1 || c.n_q_heads < 1 || c.n_kv_heads < 1 || c.max_ctx < 1)
    return CQA_ERR_INVALID_ARG;
  if (c.head_dim != 64 && c.head_dim != 128) return CQA_ERR_INVALID_ARG;
  if (c.meta_fp16 != 0 && c.meta_fp16 != 1) return CQA_ERR_INVALID_ARG;
  if (c.n_q_heads % c.n_kv_heads) return CQA_ERR_INVALID_ARG;
  const int G = c.n_q_heads / c.n_kv_heads;
  if (!(G == 1 || G == 2 || G == 4 || G == 8) || (c.head_dim == 64 && G == 8))
    return CQA_ERR_INVALID_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) return CQA_ERR_CUDA;
  if (c.device < 0 || c.device >= ndev) return CQA_ERR_INVALID_ARG;
  const int nbm = c.max_ctx / BLK;
  int smem_optin = 0;
  if (cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c.device) !=
      cudaSuccess)
    return CQA_ERR_CUDA;
  if (cqa::select_smem_bytes(G, nbm) > (size_t)smem_optin) return CQA_ERR_INVALID_ARG;

  DeviceGuard dg(c.device);
  if (!dg.ok) return CQA_ERR_CUDA;

  cqa_cache* cc = new (std::nothrow) cqa_cache();
  if (!cc) return CQA_ERR_OOM;
  cc->cfg = c;
  cc->G = G;
  cc->nbm = nbm;
  const int d = c.head_dim;
  cc->st = make_strides(nbm, d, c.max_ctx);
  const size_t units = (size_t)c.n_layers * c.batch * c.n_kv_heads;
  const size_t hq_rows = (size_t)c.batch * c.n_q_heads;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c.device) != cudaSuccess ||
      sms < 1) {
    cudaGetLastError();
    delete cc;
    return CQA_ERR_CUDA;
  }
  cc->sms = sms;
  const size_t max_chunks = (size_t)max_chunks_for(c.n_kv_heads, sms);

  // one device allocation, carved into aligned pieces
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes > 0 ? bytes : 1);
    return o;
  };
  const Strides& st = cc->st;
  const size_t o_kc = take(units * st.kcodes);
  const size_t mby = c.meta_fp16 ? 2 : 4;  // bytes of one metadata value
  const size_t o_ks = take(units * st.kscale * mby);
  const size_t o_vc = take(units * st.vcodes);
  const size_t o_vm = take(units * st.vmeta * mby);
  const size_t o_eta = take(units * st.eta * 4);
  const size_t o_vr = take(units * st.vrange * 4);
  const size_t o_kr = take(units * st.res * 2);
  const size_t o_vrs = take(units * st.res * 2);
  const size_t ls = (size_t)nbm * BLK + BLK;
  const size_t o_lg = take(hq_rows * ls * 4);
  const size_t o_e8 = take(hq_rows * nbm * 4);
  const size_t o_dl = take(hq_rows * nbm * 4);
  const size_t o_e16 = take(hq_rows * nbm * 4);
  const size_t o_er = take(hq_rows * 4);
  const size_t o_ek = take(hq_rows * 4);
  const size_t o_kst = take(hq_rows * 4);
  const size_t o_hf = take(hq_rows);
  const size_t o_bf = take((size_t)c.batch * c.n_kv_heads * nbm);
  const size_t o_dn = take(hq_rows);
  const size_t o_po = take((size_t)c.batch * c.n_kv_heads * max_chunks * G * d * 4);
  const size_t o_ps = take((size_t)c.batch * c.n_kv_heads * max_chunks * G * 3 * 4);
  const size_t o_err = take(sizeof(int));
  const size_t o_px = take((size_t)c.batch * c.n_kv_heads * max_chunks * G * 3 * 4);
  const size_t o_dcnt = take((size_t)c.batch * 2 * sizeof(int));
  const size_t o_lens = take((size_t)c.n_layers * c.batch * sizeof(int32_t));
  void* base = nullptr;
  if (cudaMalloc(&base, off) != cudaSuccess) {
    cudaGetLastError();
    delete cc;
    return CQA_ERR_OOM;
  }
  cc->dev_block = base;
  char* bp = (char*)base;
  cc->t.kcodes = (int8_t*)(bp + o_kc);
  cc->t.kscale = (float*)(bp + o_ks);
  cc->t.vcodes = (uint8_t*)(bp + o_vc);
  cc->t.vmeta = (float*)(bp + o_vm);
  cc->t.kscale_h = (__half*)(bp + o_ks);
  cc->t.vmeta_h = (__half*)(bp + o_vm);
  cc->t.meta16 = c.meta_fp16;
  cc->t.eta = (float*)(bp + o_eta);
  cc->t.vrange = (float*)(bp + o_vr);
  cc->t.kres = (__half*)(bp + o_kr);
  cc->t.vres = (__half*)(bp + o_vrs);
  cc->sc.logits = (float*)(bp + o_lg);
  cc->sc.ell8 = (float*)(bp + o_e8);
  cc->sc.delta = (float*)(bp + o_dl);
  cc->sc.ell16 = (float*)(bp + o_e16);
  cc->sc.ell_res = (float*)(bp + o_er);
  cc->sc.ekey = (float*)(bp + o_ek);
  cc->sc.kstar = (int32_t*)(bp + o_kst);
  cc->sc.hflags = (uint8_t*)(bp + o_hf);
  cc->sc.bflags = (uint8_t*)(bp + o_bf);
  cc->sc.dense = (uint8_t*)(bp + o_dn);
  cc->sc.part_o = (float*)(bp + o_po);
  cc->sc.part_s = (float*)(bp + o_ps);
  cc->sc.err = (int*)(bp + o_err);
  cc->sc.part_x = (float*)(bp + o_px);
  cc->sc.dcnt = (int*)(bp + o_dcnt);
  cc->lens_dev = (int32_t*)(bp + o_lens);
  cc->sc.ls = ls;
  cc->sc.max_chunks = (int)max_chunks;

  if (cudaMemset(base, 0, off) != cudaSuccess) {
    cqa_cache_destroy(cc);
    return CQA_ERR_CUDA;
  }
  fill_range_kernel<<<256, 256>>>(cc->t.vrange, units, d);
  if (cudaGetLastError() != cudaSuccess) {
    cqa_cache_destroy(cc);
    return CQA_ERR_CUDA;
  }

  cc->tier2_bytes = units * st.tier2 * 2;
  if (pinned_alloc(&cc->k2_host, cc->tier2_bytes, cudaHostAllocMapped | cudaHostAllocPortable) !=
          cudaSuccess ||
      pinned_alloc(&cc->v2_host, cc->tier2_bytes, cudaHostAllocMapped | cudaHostAllocPortable) !=
          cudaSuccess) {
    cudaGetLastError();
    cqa_cache_destroy(cc);
    return CQA_ERR_OOM;
  }
  void* kd = nullptr;
  void* vd = nullptr;
  if (cudaHostGetDevicePointer(&kd, cc->k2_host, 0) != cudaSuccess ||
      cudaHostGetDevicePointer(&vd, cc->v2_host, 0) != cudaSuccess) {
    cqa_cache_destroy(cc);
    return CQA_ERR_CUDA;
  }
  cc->t.k2 = (__half*)kd;
  cc->t.v2 = (__half*)vd;

  cc->len = (int32_t*)calloc((size_t)c.n_layers * c.batch, sizeof(int32_t));
  cc->seal_gen = (uint32_t*)calloc((size_t)c.n_layers, sizeof(uint32_t));
  if (!cc->len || !cc->seal_gen) {
    cqa_cache_destroy(cc);
    return CQA_ERR_OOM;
  }
  // key prefetch: two device slots of one layer's keys, a copy stream, events
  cc->pref_mode = 1;
  cc->pref_min_frac = 0.75f;
  cc->stage_layer[0] = cc->stage_layer[1] = -1;
  const size_t layer_units = (size_t)c.batch * c.n_kv_heads;
  const size_t stage_bytes = layer_units * st.tier2 * 2;
  if (cudaMalloc(&cc->kstage[0], stage_bytes) != cudaSuccess ||
      cudaMalloc(&cc->kstage[1], stage_bytes) != cudaSuccess) {
    cudaGetLastError();
    cqa_cache_destroy(cc);
    return CQA_ERR_OOM;
  }
  if (cudaStreamCreateWithFlags(&cc->side, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&cc->ev_ready[0], cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&cc->ev_ready[1], cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&cc->ev_free[0], cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&cc->ev_free[1], cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&cc->ev_main, cudaEventDisableTiming) != cudaSuccess) {
    cqa_cache_destroy(cc);
    return CQA_ERR_CUDA;
  }
  if (pinned_alloc((void**)&cc->promo_host, units * sizeof(int32_t),
                   cudaHostAllocMapped | cudaHostAllocPortable) != cudaSuccess) {
    cudaGetLastError();
    cqa_cache_destroy(cc);
    return CQA_ERR_OOM;
  }
  memset(cc->promo_host, 0xff, units * sizeof(int32_t));  // -1: no decode yet
  if (cudaHostGetDevicePointer((void**)&cc->promo_dev, cc->promo_host, 0) != cudaSuccess) {
    cqa_cache_destroy(cc);
    return CQA_ERR_CUDA;
  }
  cc->sc.promo = cc->promo_dev;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cqa_cache_destroy(cc);
    return CQA_ERR_CUDA;
  }
  *out = cc;
  return CQA_OK;
}

int cqa_cache_destroy(cqa_cache* cc) {
  if (!cc) return CQA_OK;
  int rc = CQA_OK;
  {
    DeviceGuard dg(cc->cfg.device);
    if (cudaDeviceSynchronize() != cudaSuccess) rc = CQA_ERR_CUDA;
    if (cc->dev_block) cudaFree(cc->dev_block);
    if (cc->k2_host) cudaFreeHost(cc->k2_host);
    if (cc->v2_host) cudaFreeHost(cc->v2_host);
    if (cc->prof_events)
      for (cudaEvent_t ev : *cc->prof_events) cudaEventDestroy(ev);
    for (int i = 0; i < 2; ++i) {
      if (cc->kstage[i]) cudaFree(cc->kstage[i]);
      if (cc->ev_ready[i]) cudaEventDestroy(cc->ev_ready[i]);
      if (cc->ev_free[i]) cudaEventDestroy(cc->ev_free[i]);
    }
    if (cc->ev_main) cudaEventDestroy(cc->ev_main);
    if (cc->side) cudaStreamDestroy(cc->side);
    if (cc->promo_host) cudaFreeHost(cc->promo_host);
  }
  delete cc->prof_events;
  delete cc->prof_phase;
  free(cc->len);
  free(cc->seal_gen);
  delete cc;
  return rc;
}

int cqa_cache_length(const cqa_cache* cc, int layer, int32_t* out_len) {
  if (!cc || !out_len || layer < 0 || layer >= cc->cfg.n_layers) return CQA_ERR_INVALID_ARG;
  *out_len = max_len(cc, layer);
  return CQA_OK;
}

int cqa_cache_row_lengths(const cqa_cache* cc, int layer, int32_t* out_lens) {
  if (!cc || !out_lens || layer < 0 || layer >= cc->cfg.n_layers) return CQA_ERR_INVALID_ARG;
  memcpy(out_lens, row_lens(cc, layer), (size_t)cc->cfg.batch * sizeof(int32_t));
  return CQA_OK;
}

// Append n_new tokens to `nrows` consecutive batch rows from `row0` that all
// hold T_old tokens; k, v: [nrows][n_kv_heads][n_new][head_dim].
static int append_rows(cqa_cache* cc, int layer, int row0, int nrows, const __half* kh,
                       const __half* vh, int n_new, cudaStream_t s) {
  const int B = cc->cfg.batch, Hkv = cc->cfg.n_kv_heads, d = cc->cfg.head_dim;
  int32_t* L = cc->len + (size_t)layer * B;
  const int T_old = L[row0];
  const int T_new = T_old + n_new;
  const int unit0 = (layer * B + row0) * Hkv;
  const int nb_old = T_old / BLK, nb_new = T_new / BLK;
  int32_t* lens_rows = cc->lens_dev + (size_t)layer * B + row0;
  cudaError_t e = run_phase(cc, CQA_PHASE_APPEND_SEAL, s, nb_new > nb_old ? 1 : 0, [&] {
    return launch_seal(cc->t, cc->st, unit0, nrows, Hkv, d, kh, vh, T_old, n_new, nb_old, nb_new,
                       s);
  });
  if (e == cudaSuccess)
    e = run_phase(cc, CQA_PHASE_APPEND_TAIL, s, 1, [&] {
      return launch_append_tail(cc->t, cc->st, unit0, nrows, Hkv, d, kh, vh, T_old, n_new, nb_new,
                                lens_rows, s);
    });
  if (e != cudaSuccess) return CQA_ERR_CUDA;
  for (int b = row0; b < row0 + nrows; ++b) L[b] = T_new;
  if (nb_new > nb_old) ++cc->seal_gen[layer];
  return CQA_OK;
}

int cqa_quantize_append(cqa_cache* cc, int layer, const void* k, const void* v, int n_new,
                        void* stream) {
  if (!cc || layer < 0 || layer >= cc->cfg.n_layers || n_new < 0) return CQA_ERR_INVALID_ARG;
  if (n_new == 0) return CQA_OK;
  if (!k || !v || !aligned16(k) || !aligned16(v)) return CQA_ERR_INVALID_ARG;
  if ((long long)max_len(cc, layer) + n_new > cc->cfg.max_ctx) return CQA_ERR_CAPACITY;
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok) return CQA_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const int B = cc->cfg.batch;
  const size_t row_elems = (size_t)cc->cfg.n_kv_heads * n_new * cc->cfg.head_dim;
  const __half* kh = (const __half*)k;
  const __half* vh = (const __half*)v;
  // runs of consecutive rows of equal length share one launch (all rows, when
  // the batch is not ragged)
  const int32_t* L = row_lens(cc, layer);
  for (int b0 = 0; b0 < B;) {
    int b1 = b0 + 1;
    while (b1 < B && L[b1] == L[b0]) ++b1;
    const int rc = append_rows(cc, layer, b0, b1 - b0, kh + b0 * row_elems, vh + b0 * row_elems,
                               n_new, s);
    if (rc != CQA_OK) return rc;
    b0 = b1;
  }
  return CQA_OK;
}

int cqa_quantize_append_row(cqa_cache* cc, int layer, int row, const void* k, const void* v,
                            int n_new, void* stream) {
  if (!cc || layer < 0 || layer >= cc->cfg.n_layers || row < 0 || row >= cc->cfg.batch ||
      n_new < 0)
    return CQA_ERR_INVALID_ARG;
  if (n_new == 0) return CQA_OK;
  if (!k || !v || !aligned16(k) || !aligned16(v)) return CQA_ERR_INVALID_ARG;
  if ((long long)row_lens(cc, layer)[row] + n_new > cc->cfg.max_ctx) return CQA_ERR_CAPACITY;
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok) return CQA_ERR_CUDA;
  return append_rows(cc, layer, row, 1, (const __half*)k, (const __half*)v, n_new,
                     (cudaStream_t)stream);
}

static int copy_trace(cqa_cache* cc, const DecodeShape& sh, const cqa_trace* tr, cudaStream_t s) {
  const size_t rows = (size_t)sh.B * sh.Hq;
  cudaError_t e = cudaSuccess;
  auto cp2 = [&](void* dst, const void* src, size_t elem, size_t width, size_t pitch,
                 size_t nrows) {
    if (!dst || e != cudaSuccess || width == 0) return;
    e = cudaMemcpy2DAsync(dst, width * elem, src, pitch * elem, width * elem, nrows,
                          cudaMemcpyDeviceToDevice, s);
  };
  cp2(tr->kstar, cc->sc.kstar, 4, rows, rows, 1);
  cp2(tr->head_flags, cc->sc.hflags, 1, rows, rows, 1);
  cp2(tr->ell_res, cc->sc.ell_res, 4, rows, rows, 1);
  cp2(tr->block_flags, cc->sc.bflags, 1, sh.nb_max, sh.nbm, (size_t)sh.B * sh.Hkv);
  cp2(tr->ell8, cc->sc.ell8, 4, sh.nb_max, sh.nbm, rows);
  cp2(tr->ell16, cc->sc.ell16, 4, sh.nb_max, sh.nbm, rows);
  cp2(tr->delta, cc->sc.delta, 4, sh.nb_max, sh.nbm, rows);
  return e == cudaSuccess ? CQA_OK : CQA_ERR_CUDA;
}

int cqa_decode(cqa_cache* cc, int layer, const void* q, const cqa_thresholds* th, float* out,
               float* e_key, float* e_val, uint8_t* rung, const cqa_trace* trace, void* stream) {
  if (!cc || layer < 0 || layer >= cc->cfg.n_layers || !q || !th || !out || !e_key || !e_val ||
      !rung)
    return CQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return CQA_ERR_INVALID_ARG;
  const cqa_thresholds tv = *th;
  if (!(tv.tau_cov >= 0.f) || tv.max_expand < 0 || tv.rank_r < 0 ||
      tv.rank_r > CQA_MAX_RANK_R || tv.rank_tol < 0 || isnan(tv.eps_key) ||
      isnan(tv.v_tol) || isnan(tv.eps_val) || isnan(tv.layer_dense_frac))
    return CQA_ERR_INVALID_ARG;
  if (min_len(cc, layer) == 0) return CQA_ERR_EMPTY;
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok) return CQA_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const DecodeShape sh = shape_of(cc, layer);
  if (sh.nchunks > cc->sc.max_chunks) return CQA_ERR_INVALID_ARG;
  const int unit0 = layer * sh.B * sh.Hkv;
  double need = ceil((double)tv.layer_dense_frac * sh.Hq);
  if (need < 0) need = 0;
  const int need_dense = need > 1e9 ? 1000000000 : (int)need;
  const __half* qh = (const __half*)q;
  const bool naive = tv.naive != 0;
  const bool post_check = !naive && !isinf(tv.eps_val);
  // keys of this layer staged by an earlier call, or staged now; then the next layer's
  // (a failed copy call is reported before any kernel is launched, so the
  // caller's outputs are left untouched)
  int slot = -1;
  if (!naive) {
    slot = staged_slot(cc, layer);
    if (slot < 0 && want_prefetch(cc, layer)) slot = issue_prefetch(cc, layer, -1, s);
    if (slot == -2) return CQA_ERR_CUDA;
    // the next layer's keys, copied while this layer runs: the copy shares the
    // host link with this layer's value pass, which keeps the link busy through
    // the scoring and selection phases that do not use it
    const int next = (layer + 1) % cc->cfg.n_layers;
    if (next != layer && want_prefetch(cc, next) && issue_prefetch(cc, next, slot, s) == -2)
      return CQA_ERR_CUDA;
  }
  const __half* kstage = slot >= 0 ? cc->kstage[slot] : nullptr;
  const int stage_nb = slot >= 0 ? cc->stage_nb[slot] : 0;
  if (naive) {
    // certification off: one streaming pass over Tier 1, then the split-K combine
    cudaError_t e = run_phase(cc, CQA_PHASE_NAIVE, s, 1, [&] {
      return launch_naive(cc->t, cc->st, unit0, sh, qh, cc->sc, out, e_key, e_val, rung,
                          trace != nullptr, s);
    });
    if (e == cudaSuccess)
      e = run_phase(cc, CQA_PHASE_NAIVE_COMBINE, s, 1, [&] {
        return launch_naive_combine(sh, cc->sc, out, e_key, e_val, rung, s);
      });
    if (e != cudaSuccess) return CQA_ERR_CUDA;
    if (trace) return copy_trace(cc, sh, trace, s);
    return CQA_OK;
  }
  cudaError_t e = run_phase(cc, CQA_PHASE_SCORE, s, 1,
                            [&] { return launch_score(cc->t, cc->st, unit0, sh, qh, cc->sc, s); });
  if (e == cudaSuccess)
    e = run_phase(cc, CQA_PHASE_SELECT, s, 1,
                  [&] { return launch_select(cc->t, cc->st, unit0, sh, tv, cc->sc, s); });
  if (e == cudaSuccess && slot >= 0) e = cudaStreamWaitEvent(s, cc->ev_ready[slot], 0);
  if (e == cudaSuccess && !naive && sh.nb_max > 0) {
    e = run_phase(cc, CQA_PHASE_PROMOTE, s, 1, [&] {
      return launch_promote(cc->t, cc->st, unit0, sh, qh, cc->sc, 0, kstage, stage_nb, s);
    });
    if (cc->prof_on && kstage) cc->prof_launches[CQA_PHASE_PROMOTE_STAGED] += 1;
  }
  if (e == cudaSuccess)
    e = run_phase(cc, CQA_PHASE_DECIDE, s, 1,
                  [&] { return launch_decide(sh, tv, need_dense, cc->sc, s); });
  if (e == cudaSuccess && !naive && sh.nb_max > 0)
    e = run_phase(cc, CQA_PHASE_DENSE_KEYS, s, 1, [&] {
      return launch_promote(cc->t, cc->st, unit0, sh, qh, cc->sc, 1, kstage, stage_nb, s);
    });
  if (e == cudaSuccess && slot >= 0) e = cudaEventRecord(cc->ev_free[slot], s);
  if (e == cudaSuccess)
    e = run_phase(cc, CQA_PHASE_ATTEND, s, 1,
                  [&] { return launch_attend(cc->t, cc->st, unit0, sh, qh, cc->sc, 0, s); });
  if (e == cudaSuccess)
    e = run_phase(cc, CQA_PHASE_COMBINE, s, 1, [&] {
      return launch_combine(sh, tv, cc->sc, out, e_key, e_val, rung, s);
    });
  if (e == cudaSuccess && post_check) {
    e = run_phase(cc, CQA_PHASE_DENSE_ATTEND, s, 1,
                  [&] { return launch_attend(cc->t, cc->st, unit0, sh, qh, cc->sc, 1, s); });
    if (e == cudaSuccess)
      e = run_phase(cc, CQA_PHASE_DENSE_COMBINE, s, 1, [&] {
        return launch_dense_combine(sh, cc->sc, 0, out, e_key, e_val, rung, s);
      });
  }
  if (e != cudaSuccess) return CQA_ERR_CUDA;
  if (trace) return copy_trace(cc, sh, trace, s);
  return CQA_OK;
}

int cqa_dense_reference(cqa_cache* cc, int layer, const void* q, float* out, void* stream) {
  if (!cc || layer < 0 || layer >= cc->cfg.n_layers || !q || !out) return CQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return CQA_ERR_INVALID_ARG;
  if (min_len(cc, layer) == 0) return CQA_ERR_EMPTY;
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok) return CQA_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const DecodeShape sh = shape_of(cc, layer);
  const int unit0 = layer * sh.B * sh.Hkv;
  cudaError_t e = run_phase(cc, CQA_PHASE_DENSE_ATTEND, s, 1, [&] {
    return launch_attend(cc->t, cc->st, unit0, sh, (const __half*)q, cc->sc, 2, s);
  });
  if (e == cudaSuccess)
    e = run_phase(cc, CQA_PHASE_DENSE_COMBINE, s, 1, [&] {
      return launch_dense_combine(sh, cc->sc, 1, out, nullptr, nullptr, nullptr, s);
    });
  return e == cudaSuccess ? CQA_OK : CQA_ERR_CUDA;
}

int64_t cqa_debug_export(cqa_cache* cc, int layer, int what, void* dst, size_t bytes) {
  if (!cc || layer < 0 || layer >= cc->cfg.n_layers) return CQA_ERR_INVALID_ARG;
  const int B = cc->cfg.batch, Hkv = cc->cfg.n_kv_heads, d = cc->cfg.head_dim;
  const int32_t* L = row_lens(cc, layer);
  const size_t units = (size_t)B * Hkv;
  const size_t unit0 = (size_t)layer * units;
  const Strides& st = cc->st;
  const char* srcs[2] = {nullptr, nullptr};
  size_t stride = 0;  // bytes between units
  bool host_src = false;
  int parts = 1;
  switch (what) {
    case CQA_EXPORT_KCODES: srcs[0] = (const char*)cc->t.kcodes; stride = st.kcodes; break;
    case CQA_EXPORT_KSCALE:
      srcs[0] = (const char*)cc->t.kscale;
      stride = st.kscale * (cc->t.meta16 ? 2 : 4);
      break;
    case CQA_EXPORT_VCODES: srcs[0] = (const char*)cc->t.vcodes; stride = st.vcodes; break;
    case CQA_EXPORT_VMETA:
      srcs[0] = (const char*)cc->t.vmeta;
      stride = st.vmeta * (cc->t.meta16 ? 2 : 4);
      break;
    case CQA_EXPORT_ETA: srcs[0] = (const char*)cc->t.eta; stride = st.eta * 4; break;
    case CQA_EXPORT_VRANGE: srcs[0] = (const char*)cc->t.vrange; stride = st.vrange * 4; break;
    case CQA_EXPORT_RESIDUAL:
      srcs[0] = (const char*)cc->t.kres; srcs[1] = (const char*)cc->t.vres;
      stride = st.res * 2; parts = 2;
      break;
    case CQA_EXPORT_TIER2:
      srcs[0] = (const char*)cc->k2_host; srcs[1] = (const char*)cc->v2_host;
      stride = st.tier2 * 2; parts = 2;
      host_src = true;
      break;
    default: return CQA_ERR_INVALID_ARG;
  }
  // bytes of one unit's part: each batch row exports its own extent
  auto part_bytes = [&](int T) -> size_t {
    const size_t nb = (size_t)(T / BLK), r = (size_t)(T - (T / BLK) * BLK);
    switch (what) {
      case CQA_EXPORT_KCODES: return nb * BLK * d;
      case CQA_EXPORT_KSCALE: return nb * d * 4;
      case CQA_EXPORT_VCODES: return nb * BLK * d / 2;
      case CQA_EXPORT_VMETA: return nb * BLK * (d / VG) * 8;
      case CQA_EXPORT_ETA: return nb * 4;
      case CQA_EXPORT_VRANGE: return (size_t)2 * d * 4;
      case CQA_EXPORT_RESIDUAL: return r * d * 2;
      default: return (size_t)T * d * 2;  // CQA_EXPORT_TIER2
    }
  };
  size_t total = 0;
  for (int b = 0; b < B; ++b) total += (size_t)Hkv * parts * part_bytes(L[b]);
  if (!dst && bytes == 0) return (int64_t)total;
  if (!dst || bytes != total) return CQA_ERR_INVALID_ARG;
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok || cudaDeviceSynchronize() != cudaSuccess) return CQA_ERR_CUDA;
  char* dp = (char*)dst;
  for (size_t uu = 0; uu < units; ++uu) {
    const int T = L[uu / Hkv];
    const size_t per_unit = part_bytes(T);
    for (int p = 0; p < parts; ++p, dp += per_unit) {
      const char* sp = srcs[p] + (unit0 + uu) * stride;
      if (per_unit == 0) continue;
      if (host_src) {
        // sealed tokens from Tier 2; the residual block's from device memory
        const size_t sealed = (size_t)(T / BLK) * BLK * d * 2;
        memcpy(dp, sp, sealed);
        const char* rs = (const char*)(p == 0 ? cc->t.kres : cc->t.vres) + (unit0 + uu) * st.res * 2;
        if (per_unit > sealed &&
            cudaMemcpy(dp + sealed, rs, per_unit - sealed, cudaMemcpyDeviceToHost) != cudaSuccess)
          return CQA_ERR_CUDA;
      } else if (cc->t.meta16 && (what == CQA_EXPORT_KSCALE || what == CQA_EXPORT_VMETA)) {
        // binary16 metadata: copy the halves, widen them to float32 (exact)
        const size_t n = per_unit / 4;
        std::vector<__half> tmp(n);
        if (n && cudaMemcpy(tmp.data(), sp, n * 2, cudaMemcpyDeviceToHost) != cudaSuccess)
          return CQA_ERR_CUDA;
        float* fd = (float*)dp;
        for (size_t i = 0; i < n; ++i) fd[i] = __half2float(tmp[i]);
      } else if (cudaMemcpy(dp, sp, per_unit, cudaMemcpyDeviceToHost) != cudaSuccess) {
        return CQA_ERR_CUDA;
      }
    }
  }
  return (int64_t)total;
}

int cqa_device_status(cqa_cache* cc, int32_t* status) {
  if (!cc || !status) return CQA_ERR_INVALID_ARG;
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok) return CQA_ERR_CUDA;
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return CQA_ERR_CUDA;
  if (cudaMemcpy(&v, cc->sc.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return CQA_ERR_CUDA;
  if (v) {
    // a kernel that gave up may have left its arrival counters short of zero
    if (cudaMemset(cc->sc.err, 0, sizeof(int)) != cudaSuccess ||
        cudaMemset(cc->sc.dcnt, 0, (size_t)cc->cfg.batch * 2 * sizeof(int)) != cudaSuccess)
      return CQA_ERR_CUDA;
  }
  *status = v;
  return CQA_OK;
}

int cqa_selftest_bounded_wait(cqa_cache* cc, int32_t polls) {
  if (!cc || polls < 1) return CQA_ERR_INVALID_ARG;
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok) return CQA_ERR_CUDA;
  bounded_wait_selftest_kernel<<<1, 32>>>(cc->sc.err, (uint32_t)polls);
  return cudaGetLastError() == cudaSuccess ? CQA_OK : CQA_ERR_CUDA;
}

int cqa_test_inject_fault(int site, int skip) {
  if (site < CQA_FAULT_NONE || site > CQA_FAULT_PREFETCH_COPY || skip < 0)
    return CQA_ERR_INVALID_ARG;
  g_fault_site.store(CQA_FAULT_NONE);
  g_fault_skip.store(skip);
  g_fault_site.store(site);
  return CQA_OK;
}

int cqa_set_key_prefetch(cqa_cache* cc, int mode, float min_fraction) {
  if (!cc || mode < 0 || mode > 2 || !(min_fraction >= 0.f && min_fraction <= 1.f))
    return CQA_ERR_INVALID_ARG;
  cc->pref_mode = mode;
  cc->pref_min_frac = min_fraction;
  return CQA_OK;
}

int cqa_profile_begin(cqa_cache* cc, int max_launches) {
  if (!cc || max_launches < 0) return CQA_ERR_INVALID_ARG;
  if (!cc->prof_events) {
    cc->prof_events = new (std::nothrow) std::vector<cudaEvent_t>();
    cc->prof_phase = new (std::nothrow) std::vector<int>();
    if (!cc->prof_events || !cc->prof_phase) return CQA_ERR_OOM;
  }
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok) return CQA_ERR_CUDA;
  cc->prof_phase->clear();
  cc->prof_max = (size_t)max_launches;
  cc->prof_untimed = 0;
  for (int i = 0; i < CQA_PHASE_COUNT; ++i) cc->prof_launches[i] = 0;
  cc->prof_on = true;
  return CQA_OK;
}

int cqa_profile_end(cqa_cache* cc, double* ms, int64_t* launches) {
  if (!cc || !cc->prof_on) return CQA_ERR_INVALID_ARG;
  DeviceGuard dg(cc->cfg.device);
  if (!dg.ok) return CQA_ERR_CUDA;
  cc->prof_on = false;
  double acc[CQA_PHASE_COUNT] = {0};
  for (size_t k = 0; k < cc->prof_phase->size(); ++k) {
    cudaEvent_t a = (*cc->prof_events)[2 * k], b = (*cc->prof_events)[2 * k + 1];
    if (cudaEventSynchronize(b) != cudaSuccess) return CQA_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, a, b) != cudaSuccess) return CQA_ERR_CUDA;
    acc[(*cc->prof_phase)[k]] += t;
  }
  for (int i = 0; i < CQA_PHASE_COUNT; ++i) {
    if (ms) ms[i] = acc[i];
    if (launches) launches[i] = cc->prof_launches[i];
  }
  return (int)(cc->prof_untimed > 0x7fffffff ? 0x7fffffff : cc->prof_untimed);
}

}  // extern "C"
