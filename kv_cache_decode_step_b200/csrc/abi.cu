// abi.cu -- host side of libnosa.so: the extern "C" entry points of nosa.h.
//
// The context owns every device buffer of the step (pooled keys, selection
// state, the GPU block cache and its tables, the open tail block, attention
// partials, device-side step state and statistics).  The caller owns q, the
// scores / selection / fetch buffers and the attached KV.  Every entry point
// validates, enqueues kernels on the caller's streams and returns a status.
#include <cudaTypedefs.h>

#include <climits>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/nosa.h"
#include "nosa_internal.cuh"

using namespace nosa;

namespace {

thread_local std::string g_err;

nosa_status fail(nosa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

// Injected host-side failures (nosa_debug_inject_cuda_error): the checked
// CUDA call that follows `g_inject_skip` further checked calls on this thread
// is not made and reports cudaErrorLaunchFailure.  -1: off.
thread_local int g_inject_skip = -1;

bool inject_now() {
  if (g_inject_skip < 0) return false;
  if (g_inject_skip-- > 0) return false;
  return true;  // g_inject_skip is now -1: one failure only
}

#define NOSA_CUDA(call)                                                                   \
  do {                                                                                    \
    cudaError_t e_ = inject_now() ? cudaErrorLaunchFailure : (call);                      \
    if (e_ != cudaSuccess) {                                                              \
      return fail(e_ == cudaErrorMemoryAllocation ? NOSA_ERR_NOMEM : NOSA_ERR_CUDA,       \
                  "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__,      \
                  __LINE__);                                                              \
    }                                                                                     \
  } while (0)

enum Phase { kReady = 0, kScored = 1, kSelected = 2, kFetched = 3 };

}  // namespace

void nosa::record_error(const char* msg) { g_err = msg ? msg : ""; }

// Classify a pointer: 1 device memory of this device, 2 pinned/registered
// host memory (device-addressable), 0 other.
int nosa::pointer_kind(const void* p, void** dev_ptr) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) {
    *dev_ptr = const_cast<void*>(p);
    return 1;
  }
  if (at.type == cudaMemoryTypeHost) {
    void* d = nullptr;
    if (cudaHostGetDevicePointer(&d, const_cast<void*>(p), 0) != cudaSuccess || !d) {
      cudaGetLastError();
      return 0;
    }
    *dev_ptr = d;
    return 2;
  }
  return 0;
}

struct nosa_ctx {
  nosa_config cfg{};
  int U = 0, G = 0, k = 0, C = 0, max_blocks = 0, words = 0, device = 0;
  bool offloaded = false;

  // device buffers owned by the context
  uint16_t* kbar = nullptr;
  float* agnostic = nullptr;
  int* ge = nullptr;
  int* prev = nullptr;
  uint16_t* cache_k = nullptr;
  uint16_t* cache_v = nullptr;
  int* slot_block = nullptr;
  int* last_used = nullptr;
  int* block_slot = nullptr;
  int* items = nullptr;
  int* n_hit = nullptr;
  int* n_items = nullptr;
  int4* glist = nullptr;
  uint16_t* tail_k = nullptr;
  uint16_t* tail_v = nullptr;
  float* a_pending = nullptr;
  float* part_o = nullptr;
  float2* part_ml = nullptr;
  DevState* ds = nullptr;
  DevStats* st = nullptr;
  int* refill_count = nullptr;

  // attached KV (device-addressable)
  uint16_t* kv_k = nullptr;
  uint16_t* kv_v = nullptr;
  bool attached = false;

  DecodeMaps maps{};
  bool maps_main = false;
  cudaEvent_t ev_plan = nullptr, ev_gather = nullptr;
  bool gather_on_side = false;
  cudaStream_t copy_stream = nullptr;  // given to the fetch call; the decode call runs the hits pass on it

  // host mirror of the device step state (validation only)
  int h_n_closed = 0, h_tail = 0;
  bool h_appended = false, appends_enabled = false;
  Phase phase = kReady;

  int nparts = 2, hits_parts = 2, gather_grid = 148, attn_grid = 296, hits_vpu = 1;
  int* unit_done = nullptr;
  int* done_ctr = nullptr;

  // overlapped write-through of closed blocks (KV in host memory): the close
  // kernel stages a closed block in HBM; a low-priority kernel on wt_stream
  // copies it to the host store during the next step
  uint16_t* stage_k = nullptr;
  uint16_t* stage_v = nullptr;
  cudaStream_t wt_stream = nullptr;
  cudaEvent_t ev_wt_fork = nullptr, ev_wt_done = nullptr;
  bool wt_forked = false;
  int wt_grid = 18;
  int prep_warps = 4;       // warps per CTA of the fused score/select/plan kernel
  // nosa_decode_step: a device copy of queries read from host memory, and the
  // step buffers used when the caller passes none
  uint16_t* q_dev = nullptr;
  double* own_scores = nullptr;
  int* own_sel = nullptr;
  int* own_fetch = nullptr;
  int* own_nfetch = nullptr;
  int attn_stages = 3;      // TMA stages per hits-pass CTA
  bool attn_producer = true;  // hits pass with a producer warp of its own
  bool kv_evict_first = true; // hits pass K/V loads marked first to leave L2
  bool pdl = true;            // gather placed while the plan finishes (programmatic dependent launch)
  bool placed_widen = true;   // scoring widens half of the pooled keys by bit placement
  int warm_blocks = 12;       // KV in HBM: blocks per hits-pass CTA asked of L2 during the selection
};

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// A 2-D view [rows, 128] of bf16 rows of 256 bytes, boxes of 64 rows x 64
// dims (128 bytes, the swizzle span), 128-byte swizzle.
nosa_status make_row_map(CUtensorMap* m, const void* base, unsigned long long rows) {
  auto fn = encode_fn();
  if (!fn) return fail(NOSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0) return fail(NOSA_ERR_INVALID, "KV base not 16-byte aligned");
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kP};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NOSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return NOSA_OK;
}

nosa_status validate(const nosa_config* c) {
  if (!c) return fail(NOSA_ERR_INVALID, "config is NULL");
  if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1)
    return fail(NOSA_ERR_INVALID, "batch, n_q_heads and n_kv_heads must be >= 1");
  if (c->n_q_heads % c->n_kv_heads != 0)
    return fail(NOSA_ERR_INVALID, "n_q_heads (%d) is not a multiple of n_kv_heads (%d)", c->n_q_heads,
                c->n_kv_heads);
  const int G = c->n_q_heads / c->n_kv_heads;
  if (c->head_dim != kD || c->block != kP || c->sub_block != kQ)
    return fail(NOSA_ERR_UNIMPLEMENTED, "v1 supports head_dim 128, block 64, sub_block 16 (got %d, %d, %d)",
                c->head_dim, c->block, c->sub_block);
  if (G > kMaxG) return fail(NOSA_ERR_UNIMPLEMENTED, "group size %d > %d", G, kMaxG);
  if (c->k_query < 0 || c->k_agnostic < 0 || c->k_query + c->k_agnostic < 1)
    return fail(NOSA_ERR_INVALID, "need k_query, k_agnostic >= 0 and k >= 1");
  const int k = c->k_query + c->k_agnostic;
  if (k > 256) return fail(NOSA_ERR_UNIMPLEMENTED, "budget k = %d > 256", k);
  if (c->min_overlap < 0 || c->min_overlap > k)
    return fail(NOSA_ERR_INVALID, "min_overlap %d outside [0, k=%d]", c->min_overlap, k);
  if (c->max_blocks < k || c->max_blocks > 8192)
    return fail(NOSA_ERR_INVALID, "max_blocks %d outside [k=%d, 8192]", c->max_blocks, k);
  if (c->sink_blocks < 0 || c->window_blocks < 0 || c->sink_blocks + c->window_blocks > c->k_agnostic)
    return fail(NOSA_ERR_INVALID, "need sink_blocks, window_blocks >= 0 and sink + window <= k_agnostic (%d)",
                c->k_agnostic);
  if (c->cache_slots != 0 && (c->cache_slots < k || c->cache_slots > 1024))
    return fail(NOSA_ERR_INVALID, "cache_slots %d must be 0 or in [k=%d, 1024]", c->cache_slots, k);
  const long long U = (long long)c->batch * c->n_kv_heads;
  if (U > (1 << 20)) return fail(NOSA_ERR_INVALID, "too many units");
  if (U * c->max_blocks * kP >= (1ll << 31) || U * (long long)c->cache_slots * kP >= (1ll << 31))
    return fail(NOSA_ERR_INVALID, "KV rows exceed 2^31");
  return NOSA_OK;
}

template <typename T>
nosa_status dalloc(T** p, size_t count) {
  *p = nullptr;
  if (count == 0) count = 1;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T));
  if (e != cudaSuccess) {
    *p = nullptr;
    return fail(e == cudaErrorMemoryAllocation ? NOSA_ERR_NOMEM : NOSA_ERR_CUDA, "cudaMalloc of %zu bytes: %s",
                count * sizeof(T), cudaGetErrorString(e));
  }
  return NOSA_OK;
}

void free_all(nosa_ctx* c) {
  void* ptrs[] = {c->kbar,   c->agnostic,   c->ge,        c->prev,   c->cache_k,   c->cache_v,
                  c->slot_block, c->last_used, c->block_slot, c->items, c->n_hit,   c->n_items,
                  c->glist,  c->tail_k,     c->tail_v,    c->a_pending, c->part_o, c->part_ml,
                  c->ds,     c->st,         c->refill_count, c->unit_done, c->done_ctr, c->stage_k,
                  c->stage_v, c->q_dev,  c->own_scores, c->own_sel, c->own_fetch, c->own_nfetch};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  if (c->ev_plan) cudaEventDestroy(c->ev_plan);
  if (c->ev_gather) cudaEventDestroy(c->ev_gather);
  if (c->ev_wt_fork) cudaEventDestroy(c->ev_wt_fork);
  if (c->ev_wt_done) cudaEventDestroy(c->ev_wt_done);
  if (c->wt_stream) cudaStreamDestroy(c->wt_stream);
}

WriteThroughArgs write_through_args(const nosa_ctx* c) {
  WriteThroughArgs w{};
  w.stage_k = c->stage_k;
  w.stage_v = c->stage_v;
  w.kv_k = c->kv_k;
  w.kv_v = c->kv_v;
  w.ds = c->ds;
  w.U = c->U;
  w.max_blocks = c->max_blocks;
  return w;
}

// Synchronous: lands a staged block that has not been written through yet
// (the last step closed a block) in the host store.
nosa_status flush_write_through(nosa_ctx* c) {
  if (!c->stage_k || !c->attached) return NOSA_OK;
  NOSA_CUDA(cudaDeviceSynchronize());  // the close that staged the block may still run
  NOSA_CUDA(launch_write_through(write_through_args(c), c->wt_grid, c->wt_stream));
  NOSA_CUDA(cudaStreamSynchronize(c->wt_stream));
  return NOSA_OK;
}

nosa_status set_device(nosa_ctx* c) {
  NOSA_CUDA(cudaSetDevice(c->device));
  return NOSA_OK;
}

}  // namespace

extern "C" {

const char* nosa_last_error(void) { return g_err.c_str(); }

const char* nosa_version(void) { return "nosa-b200 0.1 (sm_100a)"; }

nosa_status nosa_create(const nosa_config* cfg, nosa_ctx** out) {
  if (!out) return fail(NOSA_ERR_INVALID, "out is NULL");
  *out = nullptr;
  nosa_status s = validate(cfg);
  if (s != NOSA_OK) return s;

  nosa_ctx* c = new (std::nothrow) nosa_ctx();
  if (!c) return fail(NOSA_ERR_NOMEM, "host allocation failed");
  c->cfg = *cfg;
  c->U = cfg->batch * cfg->n_kv_heads;
  c->G = cfg->n_q_heads / cfg->n_kv_heads;
  c->k = cfg->k_query + cfg->k_agnostic;
  c->C = cfg->cache_slots;
  c->max_blocks = cfg->max_blocks;
  c->words = (cfg->max_blocks + 31) / 32;
  c->offloaded = cfg->cache_slots > 0;

  cudaError_t e = cudaGetDevice(&c->device);
  if (e != cudaSuccess) {
    delete c;
    return fail(NOSA_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c->device);
  // a quarter of the SMs keeps ~1 MiB of PCIe reads in flight, well past the
  // link's bandwidth-delay product; more CTAs only queue system-memory
  // requests that slow the attention running beside the gather
  c->gather_grid = (sms + 3) / 4;
  // fused score/select/plan: one CTA per unit; with few units, wider CTAs keep
  // about 16 warps per SM scoring (4, 8 or 16 warps per CTA)
  {
    int w = 4;
    while (w < 16 && c->U * w * 2 <= sms * 16) w *= 2;
    c->prep_warps = w;
  }
  if (const char* v = getenv("NOSA_GATHER_CTAS")) c->gather_grid = atoi(v) > 0 ? atoi(v) : c->gather_grid;
  // two persistent attention CTAs per SM, each over an equal share of the
  // (unit, block) positions; a unit's blocks span a few CTAs' shares.  With KV
  // in host memory each gather CTA's shared memory leaves room for one
  // attention CTA on its SM, so the grid shrinks to stay in one wave.
  int want = 2 * sms - (c->offloaded ? c->gather_grid : 0);
  if (want < sms) want = sms;
  if (const char* v = getenv("NOSA_ATTN_PRODUCER")) c->attn_producer = atoi(v) != 0;
  if (const char* v = getenv("NOSA_KV_EVICT_FIRST")) c->kv_evict_first = atoi(v) != 0;
  if (const char* v = getenv("NOSA_PDL")) c->pdl = atoi(v) != 0;
  if (const char* v = getenv("NOSA_PLACED_WIDEN")) c->placed_widen = atoi(v) != 0;
  if (const char* v = getenv("NOSA_WARM_BLOCKS")) c->warm_blocks = atoi(v) < 0 ? 0 : (atoi(v) > 64 ? 64 : atoi(v));
  if (const char* v = getenv("NOSA_ATTN_STAGES")) c->attn_stages = atoi(v) == 2 ? 2 : 3;
  if (c->attn_stages == 2) want = 3 * sms - (c->offloaded ? c->gather_grid : 0);
  if (const char* v = getenv("NOSA_ATTN_CTAS")) want = atoi(v) > 0 ? atoi(v) : want;
  // the hits pass walks k blocks, the open tail and kHitsGap empty positions per unit
  int gap = kHitsGap;
  if (const char* v = getenv("NOSA_ATTN_GAP")) gap = atoi(v) >= 0 && atoi(v) <= 64 ? atoi(v) : gap;
  c->hits_vpu = c->k + 1 + gap;
  c->attn_grid = attend_hits_grid(c->U, c->hits_vpu, want);
  c->hits_parts = attend_hits_parts(c->U, c->hits_vpu, c->attn_grid);
  // partial slots per unit: the hits pass's segments, then one per fetched block
  c->nparts = c->hits_parts + (c->offloaded ? c->k : 0);

  const size_t U = c->U, MB = c->max_blocks, K = c->k;
#define ALLOC(ptr, n)                    \
  do {                                   \
    s = dalloc(&(ptr), (n));             \
    if (s != NOSA_OK) {                  \
      free_all(c);                       \
      delete c;                          \
      return s;                          \
    }                                    \
  } while (0)
  ALLOC(c->kbar, U * MB * kR * kD);
  ALLOC(c->agnostic, U * MB);
  ALLOC(c->ge, U * (size_t)(cfg->k_agnostic > 0 ? cfg->k_agnostic : 1));
  ALLOC(c->prev, U * K);
  ALLOC(c->tail_k, U * kP * kD);
  ALLOC(c->tail_v, U * kP * kD);
  ALLOC(c->a_pending, U);
  ALLOC(c->part_o, U * c->nparts * c->G * kD);
  ALLOC(c->part_ml, U * c->nparts * c->G);
  ALLOC(c->ds, 1);
  ALLOC(c->st, 1);
  ALLOC(c->refill_count, 1);
  ALLOC(c->unit_done, U);
  ALLOC(c->done_ctr, 1);
  ALLOC(c->n_hit, U);
  ALLOC(c->n_items, U);
  ALLOC(c->items, U * K);
  ALLOC(c->q_dev, (size_t)cfg->batch * cfg->n_q_heads * kD);
  ALLOC(c->own_scores, U * MB);
  ALLOC(c->own_sel, U * K);
  ALLOC(c->own_fetch, U * K);
  ALLOC(c->own_nfetch, U);
  if (c->offloaded) {
    const size_t CS = c->C;
    ALLOC(c->cache_k, U * CS * kP * kD);
    ALLOC(c->cache_v, U * CS * kP * kD);
    ALLOC(c->slot_block, U * CS);
    ALLOC(c->last_used, U * CS);
    ALLOC(c->block_slot, U * MB);
    ALLOC(c->glist, U * (CS > K ? CS : K));
    ALLOC(c->stage_k, U * kP * kD);
    ALLOC(c->stage_v, U * kP * kD);
  }
#undef ALLOC
  auto cleanup = [&](nosa_status st) {
    free_all(c);
    delete c;
    return st;
  };
  if (cudaMemset(c->tail_k, 0, U * kP * kD * 2) != cudaSuccess ||
      cudaMemset(c->tail_v, 0, U * kP * kD * 2) != cudaSuccess ||
      cudaMemset(c->a_pending, 0, U * sizeof(float)) != cudaSuccess ||
      cudaMemset(c->unit_done, 0, U * sizeof(int)) != cudaSuccess ||
      cudaMemset(c->done_ctr, 0, sizeof(int)) != cudaSuccess ||
      cudaMemset(c->ds, 0, sizeof(DevState)) != cudaSuccess)
    return cleanup(fail(NOSA_ERR_CUDA, "cudaMemset failed"));
  if (cudaEventCreateWithFlags(&c->ev_plan, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_gather, cudaEventDisableTiming) != cudaSuccess)
    return cleanup(fail(NOSA_ERR_CUDA, "cudaEventCreate failed"));
  if (c->offloaded) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&c->wt_stream, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->ev_wt_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->ev_wt_done, cudaEventDisableTiming) != cudaSuccess)
      return cleanup(fail(NOSA_ERR_CUDA, "write-through stream setup failed"));
    c->wt_grid = (sms + 7) / 8;
  }
  if ((s = make_row_map(&c->maps.tk, c->tail_k, U * kP)) != NOSA_OK) return cleanup(s);
  if ((s = make_row_map(&c->maps.tv, c->tail_v, U * kP)) != NOSA_OK) return cleanup(s);
  if (c->offloaded) {
    if ((s = make_row_map(&c->maps.k, c->cache_k, U * c->C * kP)) != NOSA_OK) return cleanup(s);
    if ((s = make_row_map(&c->maps.v, c->cache_v, U * c->C * kP)) != NOSA_OK) return cleanup(s);
    c->maps_main = true;
  }
  if (configure_decode() != cudaSuccess) return cleanup(fail(NOSA_ERR_CUDA, "kernel configuration failed"));
  if (launch_reset_stats(c->st, 0) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
    return cleanup(fail(NOSA_ERR_CUDA, "initialisation failed: %s", cudaGetErrorString(cudaGetLastError())));
  *out = c;
  return NOSA_OK;
}

void nosa_destroy(nosa_ctx* ctx) {
  if (!ctx) return;
  cudaSetDevice(ctx->device);
  cudaDeviceSynchronize();
  free_all(ctx);
  delete ctx;
}

static nosa_status reset_tables(nosa_ctx* c, cudaStream_t s) {
  const size_t U = c->U;
  NOSA_CUDA(cudaMemsetAsync(c->ge, 0xFF, U * (c->cfg.k_agnostic > 0 ? c->cfg.k_agnostic : 1) * sizeof(int), s));
  NOSA_CUDA(cudaMemsetAsync(c->prev, 0xFF, U * c->k * sizeof(int), s));
  if (c->offloaded) {
    NOSA_CUDA(cudaMemsetAsync(c->slot_block, 0xFF, U * c->C * sizeof(int), s));
    NOSA_CUDA(cudaMemsetAsync(c->last_used, 0xFF, U * c->C * sizeof(int), s));
    NOSA_CUDA(cudaMemsetAsync(c->block_slot, 0xFF, U * c->max_blocks * sizeof(int), s));
  }
  return NOSA_OK;
}

nosa_status nosa_attach_kv(nosa_ctx* c, const void* k, const void* v, int n_tokens, const float* agnostic,
                           nosa_stream_t stream) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  if (!k || !v || !agnostic) return fail(NOSA_ERR_INVALID, "k, v and agnostic must be non-NULL");
  if (n_tokens < c->k * kP || n_tokens > c->max_blocks * kP)
    return fail(NOSA_ERR_INVALID, "n_tokens %d outside [k*P=%d, max_blocks*P=%d]", n_tokens, c->k * kP,
                c->max_blocks * kP);
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  // a block the previous attachment closed last still belongs in its store
  if ((s = flush_write_through(c)) != NOSA_OK) return s;
  void *dk = nullptr, *dv = nullptr, *da = nullptr;
  const int kk = pointer_kind(k, &dk), kv = pointer_kind(v, &dv), ka = pointer_kind(agnostic, &da);
  if (c->offloaded) {
    if (kk != 2 || kv != 2)
      return fail(NOSA_ERR_INVALID, "offloaded KV must be pinned host memory (cudaHostAlloc/cudaHostRegister)");
  } else if (kk != 1 || kv != 1) {
    return fail(NOSA_ERR_INVALID, "resident KV must be device memory");
  }
  if (ka != 1) return fail(NOSA_ERR_INVALID, "agnostic scores must be device memory");
  if ((reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) % 16 != 0)
    return fail(NOSA_ERR_INVALID, "KV base addresses must be 16-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t U = c->U;
  c->kv_k = static_cast<uint16_t*>(dk);
  c->kv_v = static_cast<uint16_t*>(dv);
  if (!c->offloaded) {
    if ((s = make_row_map(&c->maps.k, c->kv_k, U * c->max_blocks * kP)) != NOSA_OK) return s;
    if ((s = make_row_map(&c->maps.v, c->kv_v, U * c->max_blocks * kP)) != NOSA_OK) return s;
    c->maps_main = true;
  }
  const int n = n_tokens / kP, tail = n_tokens % kP;
  NOSA_CUDA(launch_pool(c->kv_k, (size_t)c->max_blocks * kP, c->U, 0, n * kR, c->kbar, c->max_blocks * kR, st));
  NOSA_CUDA(cudaMemcpyAsync(c->agnostic, da, U * c->max_blocks * sizeof(float), cudaMemcpyDeviceToDevice, st));
  if (tail > 0) {
    const size_t pitch_src = (size_t)c->max_blocks * kP * kD * 2;
    const size_t pitch_dst = (size_t)kP * kD * 2;
    NOSA_CUDA(cudaMemcpy2DAsync(c->tail_k, pitch_dst, c->kv_k + (size_t)n * kP * kD, pitch_src,
                                (size_t)tail * kD * 2, U, cudaMemcpyDefault, st));
    NOSA_CUDA(cudaMemcpy2DAsync(c->tail_v, pitch_dst, c->kv_v + (size_t)n * kP * kD, pitch_src,
                                (size_t)tail * kD * 2, U, cudaMemcpyDefault, st));
  }
  if ((s = reset_tables(c, st)) != NOSA_OK) return s;
  NOSA_CUDA(launch_init_state(c->ds, n, tail, 0, 0, st));
  NOSA_CUDA(cudaMemsetAsync(c->done_ctr, 0, sizeof(int), st));
  NOSA_CUDA(cudaMemsetAsync(c->unit_done, 0, U * sizeof(int), st));
  NOSA_CUDA(launch_reset_stats(c->st, st));
  c->attached = true;
  c->h_n_closed = n;
  c->h_tail = tail;
  c->h_appended = false;
  c->appends_enabled = false;
  c->phase = kReady;
  return NOSA_OK;
}

nosa_status nosa_append_token(nosa_ctx* c, const void* k_new, const void* v_new, const float* a_close,
                              nosa_stream_t stream) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  if (!c->attached) return fail(NOSA_ERR_ORDER, "append before attach");
  if (c->phase != kReady || c->h_appended) return fail(NOSA_ERR_ORDER, "append must come first in a step, once");
  if (!k_new || !v_new) return fail(NOSA_ERR_INVALID, "k_new and v_new must be non-NULL");
  if (c->h_tail + 1 > kP || c->h_n_closed * kP + c->h_tail + 1 > c->max_blocks * kP)
    return fail(NOSA_ERR_INVALID, "append beyond max_blocks*P tokens");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  AppendArgs a{};
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  a.a_close = a_close;
  a.tail_k = c->tail_k;
  a.tail_v = c->tail_v;
  a.a_pending = c->a_pending;
  a.ds = c->ds;
  a.U = c->U;
  a.max_blocks = c->max_blocks;
  NOSA_CUDA(launch_append(a, reinterpret_cast<cudaStream_t>(stream)));
  c->h_tail += 1;
  c->h_appended = true;
  c->appends_enabled = true;
  return NOSA_OK;
}

namespace {

ScoreArgs score_args(const nosa_ctx* c, const void* q, double* scores) {
  ScoreArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.kbar = c->kbar;
  a.scores = scores;
  a.ds = c->ds;
  a.U = c->U;
  a.Hq = c->cfg.n_q_heads;
  a.Hkv = c->cfg.n_kv_heads;
  a.G = c->G;
  a.max_blocks = c->max_blocks;
  a.placed_widen = c->placed_widen ? 1 : 0;
  return a;
}

SelectArgs select_args(const nosa_ctx* c, const double* scores, int32_t* sel) {
  SelectArgs a{};
  a.agnostic = c->agnostic;
  a.scores = scores;
  a.ge = c->ge;
  a.prev = c->prev;
  a.sel = sel;
  a.ds = c->ds;
  a.st = c->st;
  a.U = c->U;
  a.max_blocks = c->max_blocks;
  a.k_q = c->cfg.k_query;
  a.k_e = c->cfg.k_agnostic;
  a.k = c->k;
  a.c_max = c->k - c->cfg.min_overlap;
  a.words = c->words;
  a.sink = c->cfg.sink_blocks;
  a.window = c->cfg.window_blocks;
  return a;
}

PlanArgs plan_args(const nosa_ctx* c, const int32_t* sel, int32_t* fetch, int32_t* n_fetch) {
  PlanArgs p{};
  p.sel = sel;
  p.fetch = fetch;
  p.n_fetch = n_fetch;
  p.slot_block = c->slot_block;
  p.last_used = c->last_used;
  p.block_slot = c->block_slot;
  p.items = c->items;
  p.n_hit = c->n_hit;
  p.n_items = c->n_items;
  p.glist = c->glist;
  p.ds = c->ds;
  p.st = c->st;
  p.U = c->U;
  p.k = c->k;
  p.C = c->C;
  p.max_blocks = c->max_blocks;
  return p;
}

// A block closed by the previous step goes to the host store while this step
// runs; nosa_sparse_decode joins it before the next close.
nosa_status fork_write_through(nosa_ctx* c, cudaStream_t st) {
  if (!(c->stage_k && c->appends_enabled)) return NOSA_OK;
  NOSA_CUDA(cudaEventRecord(c->ev_wt_fork, st));
  NOSA_CUDA(cudaStreamWaitEvent(c->wt_stream, c->ev_wt_fork, 0));
  NOSA_CUDA(launch_write_through(write_through_args(c), c->wt_grid, c->wt_stream));
  NOSA_CUDA(cudaEventRecord(c->ev_wt_done, c->wt_stream));
  c->wt_forked = true;
  return NOSA_OK;
}

}  // namespace

nosa_status nosa_score_blocks(nosa_ctx* c, const void* q, double* scores, nosa_stream_t stream) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  if (!c->attached) return fail(NOSA_ERR_ORDER, "score before attach");
  if (c->phase != kReady) return fail(NOSA_ERR_ORDER, "score must start a step (after decode or append)");
  if (!q || !scores) return fail(NOSA_ERR_INVALID, "q and scores must be non-NULL");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((s = fork_write_through(c, st)) != NOSA_OK) return s;
  NOSA_CUDA(launch_score(score_args(c, q, scores), st));
  c->phase = kScored;
  return NOSA_OK;
}

nosa_status nosa_select(nosa_ctx* c, const double* scores, int32_t* sel, nosa_stream_t stream) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  if (c->phase != kScored) return fail(NOSA_ERR_ORDER, "select must follow score");
  if (!scores || !sel) return fail(NOSA_ERR_INVALID, "scores and sel must be non-NULL");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  NOSA_CUDA(launch_select(select_args(c, scores, sel), reinterpret_cast<cudaStream_t>(stream)));
  c->phase = kSelected;
  return NOSA_OK;
}

nosa_status nosa_fetch_missing(nosa_ctx* c, const int32_t* sel, int32_t* fetch, int32_t* n_fetch,
                               nosa_stream_t compute, nosa_stream_t copy) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  if (c->phase != kSelected) return fail(NOSA_ERR_ORDER, "fetch must follow select");
  if (!sel || !fetch || !n_fetch) return fail(NOSA_ERR_INVALID, "sel, fetch and n_fetch must be non-NULL");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(compute);
  cudaStream_t xs = reinterpret_cast<cudaStream_t>(copy);
  if (!c->offloaded) {
    NOSA_CUDA(cudaMemsetAsync(fetch, 0xFF, (size_t)c->U * c->k * sizeof(int32_t), cs));
    NOSA_CUDA(cudaMemsetAsync(n_fetch, 0, (size_t)c->U * sizeof(int32_t), cs));
    c->gather_on_side = false;
    c->phase = kFetched;
    return NOSA_OK;
  }
  NOSA_CUDA(launch_plan(plan_args(c, sel, fetch, n_fetch), cs));
  c->copy_stream = xs;
  c->gather_on_side = (xs != cs);
  c->phase = kFetched;
  return NOSA_OK;
}

namespace {

// The fused first half of a step.  q_copy: null (q is device memory), or the
// context's device copy that the kernel fills while it reads q once from
// (mapped) host memory.
nosa_status fused_first_half(nosa_ctx* c, const void* q, uint16_t* q_copy, double* scores, int32_t* sel,
                             int32_t* fetch, int32_t* n_fetch, nosa_stream_t compute, nosa_stream_t copy) {
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(compute);
  cudaStream_t xs = reinterpret_cast<cudaStream_t>(copy);
  if ((s = fork_write_through(c, cs)) != NOSA_OK) return s;
  PrepareArgs a{};
  a.sc = score_args(c, q, scores);
  a.sc.q_copy = q_copy;
  a.se = select_args(c, scores, sel);
  a.pl = plan_args(c, sel, fetch, n_fetch);
  a.offloaded = c->offloaded ? 1 : 0;
  a.nwarps = c->prep_warps;
  if (!c->offloaded && c->warm_blocks > 0) {
    a.warm_k = c->kv_k;
    a.warm_v = c->kv_v;
    a.warm_blocks = c->warm_blocks;
    a.hits_vpu = c->hits_vpu;
    a.hits_grid = c->attn_grid;
  }
  NOSA_CUDA(launch_prepare(a, cs));
  c->copy_stream = xs;
  c->gather_on_side = c->offloaded && xs != cs;
  c->phase = kFetched;
  return NOSA_OK;
}

}  // namespace

nosa_status nosa_score_select_fetch(nosa_ctx* c, const void* q, double* scores, int32_t* sel, int32_t* fetch,
                                    int32_t* n_fetch, nosa_stream_t compute, nosa_stream_t copy) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  if (!c->attached) return fail(NOSA_ERR_ORDER, "score before attach");
  if (c->phase != kReady) return fail(NOSA_ERR_ORDER, "score must start a step (after decode or append)");
  if (!q || !scores || !sel || !fetch || !n_fetch)
    return fail(NOSA_ERR_INVALID, "q, scores, sel, fetch and n_fetch must be non-NULL");
  if (!prepare_supported(c->max_blocks)) {
    // beyond the fused kernel's block count: scores from the scoring grid,
    // then selection and plan in one launch (up to 1024 blocks per unit), or
    // the three calls in a row
    nosa_status s = nosa_score_blocks(c, q, scores, compute);
    if (s != NOSA_OK) return s;
    if (!select_plan_supported(c->max_blocks)) {
      s = nosa_select(c, scores, sel, compute);
      if (s == NOSA_OK) s = nosa_fetch_missing(c, sel, fetch, n_fetch, compute, copy);
      return s;
    }
    NOSA_CUDA(launch_select_plan(select_args(c, scores, sel), plan_args(c, sel, fetch, n_fetch), c->offloaded ? 1 : 0,
                                 reinterpret_cast<cudaStream_t>(compute), c->pdl));
    c->copy_stream = reinterpret_cast<cudaStream_t>(copy);
    c->gather_on_side = c->offloaded && copy != compute;
    c->phase = kFetched;
    return NOSA_OK;
  }
  return fused_first_half(c, q, nullptr, scores, sel, fetch, n_fetch, compute, copy);
}

nosa_status nosa_decode_step(nosa_ctx* c, const void* q, double* scores, int32_t* sel, int32_t* fetch,
                             int32_t* n_fetch, void* out, nosa_stream_t compute, nosa_stream_t copy) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  if (!c->attached) return fail(NOSA_ERR_ORDER, "step before attach");
  if (c->phase != kReady) return fail(NOSA_ERR_ORDER, "a step starts after decode or append");
  if (!q || !out) return fail(NOSA_ERR_INVALID, "q and out must be non-NULL");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  void *qd = nullptr, *od = nullptr;
  const int qk = pointer_kind(q, &qd), ok = pointer_kind(out, &od);
  if (qk == 0 || ok == 0) return fail(NOSA_ERR_INVALID, "q and out must be device or pinned host memory");
  if ((reinterpret_cast<uintptr_t>(qd) | reinterpret_cast<uintptr_t>(od)) % 16 != 0)
    return fail(NOSA_ERR_INVALID, "q and out must be 16-byte aligned");
  if (!scores) scores = c->own_scores;
  if (!sel) sel = c->own_sel;
  if (!fetch) fetch = c->own_fetch;
  if (!n_fetch) n_fetch = c->own_nfetch;
  const void* q_attn = qd;  // the queries the attention reads: device memory
  if (qk == 2) {
    q_attn = c->q_dev;
    if (prepare_supported(c->max_blocks)) {
      s = fused_first_half(c, qd, c->q_dev, scores, sel, fetch, n_fetch, compute, copy);
    } else {
      // beyond the fused kernel's block count: one copy in, then the three calls
      NOSA_CUDA(cudaMemcpyAsync(c->q_dev, q, (size_t)c->cfg.batch * c->cfg.n_q_heads * kD * 2,
                                cudaMemcpyHostToDevice, reinterpret_cast<cudaStream_t>(compute)));
      s = nosa_score_select_fetch(c, c->q_dev, scores, sel, fetch, n_fetch, compute, copy);
    }
  } else {
    s = nosa_score_select_fetch(c, qd, scores, sel, fetch, n_fetch, compute, copy);
  }
  if (s != NOSA_OK) return s;
  return nosa_sparse_decode(c, q_attn, sel, od, compute);
}

nosa_status nosa_sparse_decode(nosa_ctx* c, const void* q, const int32_t* sel, void* out, nosa_stream_t stream) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  if (!(c->phase == kFetched || (!c->offloaded && c->phase == kSelected)))
    return fail(NOSA_ERR_ORDER, "decode must follow fetch (or select when KV is resident)");
  if (!q || !sel || !out) return fail(NOSA_ERR_INVALID, "q, sel and out must be non-NULL");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.sel = sel;
  a.items = c->items;
  a.n_hit = c->n_hit;
  a.n_items = c->n_items;
  a.part_o = c->part_o;
  a.part_ml = c->part_ml;
  a.ds = c->ds;
  a.U = c->U;
  a.Hq = c->cfg.n_q_heads;
  a.Hkv = c->cfg.n_kv_heads;
  a.G = c->G;
  a.k = c->k;
  a.max_blocks = c->max_blocks;
  a.C = c->C;
  a.resident = c->offloaded ? 0 : 1;
  a.tail_split = 1;
  a.vpu = c->hits_vpu;
  a.nparts = c->nparts;
  a.part_base = 0;
  a.hits_grid = c->attn_grid;
  a.kv_evict_first = c->kv_evict_first ? 1 : 0;
  a.out = static_cast<uint16_t*>(out);
  a.st = c->st;
  a.miss_base = c->hits_parts;
  // Every unit's partials are counted in unit_done; whichever kernel completes
  // a unit merges it, and without a block close to follow, the last unit
  // merged ends the step itself (no advance launch).
  const bool fold_advance = !c->appends_enabled;
  a.unit_done = c->unit_done;
  a.done_ctr = fold_advance ? c->done_ctr : nullptr;
  if (c->offloaded) {
    // the misses: copied from host memory into their cache slots and attended
    // as they land, on the copy stream given to the fetch call, beside the
    // hits pass
    GatherAttendArgs ga{};
    ga.g.hk = c->kv_k;
    ga.g.hv = c->kv_v;
    ga.g.ck = c->cache_k;
    ga.g.cv = c->cache_v;
    ga.g.glist = c->glist;
    ga.g.count = &c->ds->gather_count;
    ga.g.stage_k = c->stage_k;
    ga.g.stage_v = c->stage_v;
    ga.g.ds = c->ds;
    ga.g.U = c->U;
    ga.g.C = c->C;
    ga.g.max_blocks = c->max_blocks;
    ga.d = a;
    if (c->gather_on_side) {
      // the gather goes first, on this stream, so its CTAs are placed before
      // the hits pass's; the hits pass runs beside it on the second stream
      NOSA_CUDA(cudaEventRecord(c->ev_plan, st));
      NOSA_CUDA(launch_gather_attend(ga, c->gather_grid, st, c->pdl));
      NOSA_CUDA(cudaStreamWaitEvent(c->copy_stream, c->ev_plan, 0));
      NOSA_CUDA(launch_attend_hits(a, c->maps, c->attn_grid, c->copy_stream, c->attn_stages, c->attn_producer));
      NOSA_CUDA(cudaEventRecord(c->ev_gather, c->copy_stream));
      NOSA_CUDA(cudaStreamWaitEvent(st, c->ev_gather, 0));
    } else {
      NOSA_CUDA(launch_gather_attend(ga, c->gather_grid, st, c->pdl));
    }
  }
  // hits pass: blocks already on the GPU (all of S(t) when KV is in HBM) plus
  // the open tail
  if (!c->gather_on_side)
    NOSA_CUDA(launch_attend_hits(a, c->maps, c->attn_grid, st, c->attn_stages, c->attn_producer));
  if (c->appends_enabled) {
    CloseArgs cl{};
    cl.tail_k = c->tail_k;
    cl.tail_v = c->tail_v;
    cl.a_pending = c->a_pending;
    cl.kbar = c->kbar;
    cl.agnostic = c->agnostic;
    cl.kv_k = c->kv_k;
    cl.kv_v = c->kv_v;
    cl.stage_k = c->stage_k;
    cl.stage_v = c->stage_v;
    cl.ds = c->ds;
    cl.U = c->U;
    cl.max_blocks = c->max_blocks;
    if (c->wt_forked) {
      NOSA_CUDA(cudaStreamWaitEvent(st, c->ev_wt_done, 0));
      c->wt_forked = false;
    }
    NOSA_CUDA(launch_close(cl, st));
  }
  if (!fold_advance) NOSA_CUDA(launch_advance(c->ds, c->st, st));
  if (c->h_tail >= kP) {
    c->h_n_closed += 1;
    c->h_tail = 0;
  }
  c->h_appended = false;
  c->phase = kReady;
  return NOSA_OK;
}

nosa_status nosa_get_stats(nosa_ctx* c, nosa_stats* out) {
  if (!c || !out) return fail(NOSA_ERR_INVALID, "ctx and stats must be non-NULL");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  NOSA_CUDA(cudaDeviceSynchronize());
  DevStats h{};
  DevState d{};
  NOSA_CUDA(cudaMemcpy(&h, c->st, sizeof h, cudaMemcpyDeviceToHost));
  NOSA_CUDA(cudaMemcpy(&d, c->ds, sizeof d, cudaMemcpyDeviceToHost));
  memset(out, 0, sizeof *out);
  out->steps = (int64_t)h.steps;
  out->selected = (int64_t)h.selected;
  out->hits = (int64_t)h.hits;
  out->misses = (int64_t)h.misses;
  out->fetched_bytes = (int64_t)h.fetched_bytes;
  out->overlap_sum = (int64_t)h.overlap_sum;
  out->overlap_terms = (int64_t)h.overlap_terms;
  out->min_overlap = h.min_overlap;
  out->max_fetch = h.max_fetch;
  out->error_bits = d.error_bits;
  out->n_closed = d.n_closed;
  out->tail_len = d.tail_len;
  return NOSA_OK;
}

nosa_status nosa_reset_stats(nosa_ctx* c, nosa_stream_t stream) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  NOSA_CUDA(launch_reset_stats(c->st, reinterpret_cast<cudaStream_t>(stream)));
  return NOSA_OK;
}

nosa_status nosa_check_errors(nosa_ctx* c) {
  if (!c) return fail(NOSA_ERR_INVALID, "ctx is NULL");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  NOSA_CUDA(cudaDeviceSynchronize());
  DevState d{};
  NOSA_CUDA(cudaMemcpy(&d, c->ds, sizeof d, cudaMemcpyDeviceToHost));
  if (d.error_bits & ERR_TIMEOUT) return fail(NOSA_ERR_TIMEOUT, "a bounded device wait ran out (bits 0x%x)", d.error_bits);
  if (d.error_bits) return fail(NOSA_ERR_INVALID, "device-side check failed (bits 0x%x)", d.error_bits);
  return NOSA_OK;
}

nosa_status nosa_read_cache_map(nosa_ctx* c, int32_t* slot_block) {
  if (!c || !slot_block) return fail(NOSA_ERR_INVALID, "ctx and slot_block must be non-NULL");
  if (!c->offloaded) return fail(NOSA_ERR_INVALID, "KV is resident: there is no cache");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  NOSA_CUDA(cudaDeviceSynchronize());
  NOSA_CUDA(cudaMemcpy(slot_block, c->slot_block, (size_t)c->U * c->C * sizeof(int), cudaMemcpyDeviceToHost));
  return NOSA_OK;
}

nosa_status nosa_read_cache(nosa_ctx* c, int unit_begin, int n_units, void* k_host, void* v_host) {
  if (!c || !k_host || !v_host) return fail(NOSA_ERR_INVALID, "ctx, k_host and v_host must be non-NULL");
  if (!c->offloaded) return fail(NOSA_ERR_INVALID, "KV is resident: there is no cache");
  if (unit_begin < 0 || n_units < 0 || unit_begin + (long long)n_units > c->U)
    return fail(NOSA_ERR_INVALID, "units [%d, %d + %d) outside [0, %d)", unit_begin, unit_begin, n_units, c->U);
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  NOSA_CUDA(cudaDeviceSynchronize());
  const size_t per_unit = (size_t)c->C * kP * kD;  // bf16 elements of one unit's slots
  const size_t bytes = per_unit * n_units * sizeof(uint16_t);
  NOSA_CUDA(cudaMemcpy(k_host, c->cache_k + per_unit * unit_begin, bytes, cudaMemcpyDeviceToHost));
  NOSA_CUDA(cudaMemcpy(v_host, c->cache_v + per_unit * unit_begin, bytes, cudaMemcpyDeviceToHost));
  return NOSA_OK;
}

// ---------------------------------------------------------------- checkpoint
namespace {
struct StateHeader {
  uint32_t magic, version;
  int32_t U, k, k_e, C, max_blocks, G;
};
constexpr uint32_t kMagic = 0x4E4F5341u;  // "NOSA"

size_t state_size(const nosa_ctx* c) {
  const size_t U = c->U, KE = c->cfg.k_agnostic > 0 ? c->cfg.k_agnostic : 1;
  size_t n = sizeof(StateHeader) + sizeof(DevState);
  n += U * KE * 4 + U * c->k * 4;                         // ge, prev
  n += U * c->max_blocks * 4;                             // agnostic
  n += U * 4;                                             // a_pending
  n += 2 * U * kP * kD * 2;                               // tail K, V
  if (c->offloaded) n += 2 * U * c->C * 4 + U * c->max_blocks * 4;  // slot_block, last_used, block_slot
  return n;
}
}  // namespace

nosa_status nosa_get_state(nosa_ctx* c, void* buf, size_t* size) {
  if (!c || !size) return fail(NOSA_ERR_INVALID, "ctx and size must be non-NULL");
  const size_t need = state_size(c);
  if (!buf) {
    *size = need;
    return NOSA_OK;
  }
  if (*size < need) return fail(NOSA_ERR_INVALID, "buffer of %zu bytes < %zu", *size, need);
  if (!c->attached) return fail(NOSA_ERR_ORDER, "get_state before attach");
  if (c->phase != kReady) return fail(NOSA_ERR_ORDER, "get_state only between steps");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  NOSA_CUDA(cudaDeviceSynchronize());
  if ((s = flush_write_through(c)) != NOSA_OK) return s;
  unsigned char* p = static_cast<unsigned char*>(buf);
  StateHeader h{kMagic, 2u, c->U, c->k, c->cfg.k_agnostic, c->C, c->max_blocks, c->G};
  memcpy(p, &h, sizeof h);
  p += sizeof h;
  const size_t U = c->U, KE = c->cfg.k_agnostic > 0 ? c->cfg.k_agnostic : 1;
  auto get = [&](const void* dev, size_t bytes) -> nosa_status {
    NOSA_CUDA(cudaMemcpy(p, dev, bytes, cudaMemcpyDeviceToHost));
    p += bytes;
    return NOSA_OK;
  };
  if ((s = get(c->ds, sizeof(DevState))) != NOSA_OK) return s;
  if ((s = get(c->ge, U * KE * 4)) != NOSA_OK) return s;
  if ((s = get(c->prev, U * c->k * 4)) != NOSA_OK) return s;
  if ((s = get(c->agnostic, U * c->max_blocks * 4)) != NOSA_OK) return s;
  if ((s = get(c->a_pending, U * 4)) != NOSA_OK) return s;
  if ((s = get(c->tail_k, U * kP * kD * 2)) != NOSA_OK) return s;
  if ((s = get(c->tail_v, U * kP * kD * 2)) != NOSA_OK) return s;
  if (c->offloaded) {
    if ((s = get(c->slot_block, U * c->C * 4)) != NOSA_OK) return s;
    if ((s = get(c->last_used, U * c->C * 4)) != NOSA_OK) return s;
    if ((s = get(c->block_slot, U * c->max_blocks * 4)) != NOSA_OK) return s;
  }
  *size = need;
  return NOSA_OK;
}

nosa_status nosa_set_state(nosa_ctx* c, const void* buf, size_t size) {
  if (!c || !buf) return fail(NOSA_ERR_INVALID, "ctx and buf must be non-NULL");
  if (!c->attached) return fail(NOSA_ERR_ORDER, "set_state before attach");
  if (c->phase != kReady) return fail(NOSA_ERR_ORDER, "set_state only between steps");
  const size_t need = state_size(c);
  if (size != need) return fail(NOSA_ERR_INVALID, "state blob of %zu bytes, expected %zu", size, need);
  StateHeader h;
  memcpy(&h, buf, sizeof h);
  if (h.magic != kMagic || h.version != 2u || h.U != c->U || h.k != c->k || h.k_e != c->cfg.k_agnostic ||
      h.C != c->C || h.max_blocks != c->max_blocks || h.G != c->G)
    return fail(NOSA_ERR_INVALID, "state blob from a different configuration");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  NOSA_CUDA(cudaDeviceSynchronize());
  if ((s = flush_write_through(c)) != NOSA_OK) return s;
  const unsigned char* p = static_cast<const unsigned char*>(buf) + sizeof h;
  DevState d;
  memcpy(&d, p, sizeof d);
  if (d.n_closed < 0 || d.n_closed > c->max_blocks || d.tail_len < 0 || d.tail_len >= kP)
    return fail(NOSA_ERR_INVALID, "state blob holds an invalid block count");
  // the blob was taken after a write-through flush: every closed block is in
  // the attached store and nothing is staged in this context
  d.staged_block = -1;
  d.wt_block = -1;
  d.wt_done = 0;
  d.gather_next = 0;
  const size_t U = c->U, KE = c->cfg.k_agnostic > 0 ? c->cfg.k_agnostic : 1;
  auto put = [&](void* dev, size_t bytes) -> nosa_status {
    NOSA_CUDA(cudaMemcpy(dev, p, bytes, cudaMemcpyHostToDevice));
    p += bytes;
    return NOSA_OK;
  };
  NOSA_CUDA(cudaMemcpy(c->ds, &d, sizeof d, cudaMemcpyHostToDevice));
  p += sizeof d;
  if ((s = put(c->ge, U * KE * 4)) != NOSA_OK) return s;
  if ((s = put(c->prev, U * c->k * 4)) != NOSA_OK) return s;
  if ((s = put(c->agnostic, U * c->max_blocks * 4)) != NOSA_OK) return s;
  if ((s = put(c->a_pending, U * 4)) != NOSA_OK) return s;
  if ((s = put(c->tail_k, U * kP * kD * 2)) != NOSA_OK) return s;
  if ((s = put(c->tail_v, U * kP * kD * 2)) != NOSA_OK) return s;
  std::vector<int4> refill;
  if (c->offloaded) {
    std::vector<int> sb(U * c->C);
    memcpy(sb.data(), p, sb.size() * 4);
    for (size_t u = 0; u < U; ++u)
      for (int slot = 0; slot < c->C; ++slot) {
        const int b = sb[u * c->C + slot];
        if (b >= 0 && b < c->max_blocks) refill.push_back(make_int4((int)u, b, slot, 0));
      }
    if ((s = put(c->slot_block, U * c->C * 4)) != NOSA_OK) return s;
    if ((s = put(c->last_used, U * c->C * 4)) != NOSA_OK) return s;
    if ((s = put(c->block_slot, U * c->max_blocks * 4)) != NOSA_OK) return s;
  }
  // rebuild pooled keys of the closed blocks from the attached KV and refill
  // the cache slots from the host copy
  NOSA_CUDA(launch_pool(c->kv_k, (size_t)c->max_blocks * kP, c->U, 0, d.n_closed * kR, c->kbar,
                        c->max_blocks * kR, 0));
  if (!refill.empty()) {
    int4* dl = nullptr;
    NOSA_CUDA(cudaMalloc(&dl, refill.size() * sizeof(int4)));
    const int cnt = (int)refill.size();
    cudaError_t e = cudaMemcpy(dl, refill.data(), refill.size() * sizeof(int4), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(c->refill_count, &cnt, sizeof cnt, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) {
      GatherArgs g{};
      g.hk = c->kv_k;
      g.hv = c->kv_v;
      g.ck = c->cache_k;
      g.cv = c->cache_v;
      g.glist = dl;
      g.count = c->refill_count;
      g.ds = c->ds;
      g.U = c->U;
      g.C = c->C;
      g.max_blocks = c->max_blocks;
      e = launch_gather(g, c->gather_grid, 0);
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    cudaFree(dl);
    if (e != cudaSuccess) return fail(NOSA_ERR_CUDA, "cache refill failed: %s", cudaGetErrorString(e));
  }
  NOSA_CUDA(cudaDeviceSynchronize());
  c->h_n_closed = d.n_closed;
  c->h_tail = d.tail_len;
  c->h_appended = false;
  c->appends_enabled = c->appends_enabled || d.tail_len > 0;
  c->phase = kReady;
  return NOSA_OK;
}

nosa_status nosa_debug_inject_cuda_error(int skip) {
  if (skip < -1) return fail(NOSA_ERR_INVALID, "skip must be >= -1");
  g_inject_skip = skip;
  return NOSA_OK;
}

nosa_status nosa_debug_wait_flag(nosa_ctx* c, const int32_t* flag, int timeout_ms, nosa_stream_t stream) {
  if (!c || !flag) return fail(NOSA_ERR_INVALID, "ctx and flag must be non-NULL");
  if (timeout_ms < 0 || timeout_ms > 10000) return fail(NOSA_ERR_INVALID, "timeout_ms must be in [0, 10000]");
  nosa_status s = set_device(c);
  if (s != NOSA_OK) return s;
  void* dp = nullptr;
  const int kind = pointer_kind(flag, &dp);
  if (kind == 0) return fail(NOSA_ERR_INVALID, "flag must be device or pinned host memory");
  NOSA_CUDA(launch_wait_flag(static_cast<const volatile int*>(dp), c->ds, (long long)timeout_ms * 1000000ll,
                             reinterpret_cast<cudaStream_t>(stream)));
  return NOSA_OK;
}

}  // extern "C"
