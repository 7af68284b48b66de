// noalloc.cu -- block-sparse attention for callers that cannot allocate
// device memory.
//
// Some embedders of this library cannot call cudaMalloc: a serving engine that
// reserves nearly all of HBM up front for its own pool allocator leaves no room
// for a library's private buffers, and code that is not allowed to introduce
// device-wide synchronisation (cudaMalloc / cudaFree may synchronise) cannot
// create a context either.  nosa_sparse_decode_noalloc serves them: it runs the
// same split-KV attention kernels as nosa_sparse_decode over a resident KV
// store, but keeps the split partials in a fixed-size array that lives in the
// library image itself, so the call allocates nothing.
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "../../include/nosa.h"
#include "nosa_internal.cuh"

namespace nosa {

// Capacity of the shared scratch: partial rows of (128 fp32 accumulators) plus
// one (max, sum) pair each, and one merge counter per unit.  A call with U
// units of G query heads needs U * G * (ceil(grid / U) + 1) rows for a grid of
// at most 2 CTAs per SM; that fits whenever U * G = B * H_q <= kNoAllocHeads.
constexpr int kNoAllocRows = 16384;
constexpr int kNoAllocHeads = 8192;

// File-scope scratch, held by every GPU that loads the library until exit.
// Host code must not use these names as device addresses; it takes their
// device addresses with cudaGetSymbolAddress (see device_scratch below).
static __device__ __align__(256) float g_noalloc_part_o[kNoAllocRows * kD];
static __device__ __align__(256) float2 g_noalloc_part_ml[kNoAllocRows];
static __device__ __align__(256) DevState g_noalloc_state;
static __device__ __align__(256) int g_noalloc_unit_done[kNoAllocRows];

namespace {

constexpr int kMaxDevices = 64;

struct DeviceScratch {
  bool ready = false;
  float* part_o = nullptr;
  float2* part_ml = nullptr;
  DevState* state = nullptr;
  int* unit_done = nullptr;
};

DeviceScratch g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// Failures are reported through nosa_last_error(), like every other call.
nosa_status noalloc_fail(nosa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  record_error(buf);
  return s;
}

// Once per device, with that device current: resolve the device addresses of
// the scratch arrays and configure the attention kernel's shared memory.
nosa_status device_scratch(int dev, DeviceScratch** out) {
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(NOSA_ERR_INVALID, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceScratch& d = g_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_part_o);
    if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    d.part_o = static_cast<float*>(p);
    e = cudaGetSymbolAddress(&p, g_noalloc_part_ml);
    if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    d.part_ml = static_cast<float2*>(p);
    e = cudaGetSymbolAddress(&p, g_noalloc_state);
    if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    d.state = static_cast<DevState*>(p);
    e = cudaGetSymbolAddress(&p, g_noalloc_unit_done);
    if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    d.unit_done = static_cast<int*>(p);
    e = configure_decode();
    if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "kernel configuration: %s", cudaGetErrorString(e));
    d.ready = true;
  }
  *out = &d;
  return NOSA_OK;
}

// 2-D TMA view [rows, 128] of bf16 rows, 64 x 64 boxes, 128-byte swizzle.  Fills a
// host-side descriptor; allocates nothing.
nosa_status encode_rows(CUtensorMap* m, const void* base, unsigned long long rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return noalloc_fail(NOSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kP};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return noalloc_fail(NOSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return NOSA_OK;
}

}  // namespace
}  // namespace nosa

using namespace nosa;

extern "C" {

NOSA_API nosa_status nosa_sparse_decode_noalloc(const void* q, const void* k, const void* v, int batch,
                                                int n_q_heads, int n_kv_heads, int max_blocks,
                                                const int32_t* sel, int k_sel, void* out,
                                                nosa_stream_t stream) {
  if (!q || !k || !v || !sel || !out) return noalloc_fail(NOSA_ERR_INVALID, "NULL argument");
  if (batch < 1 || n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads != 0)
    return noalloc_fail(NOSA_ERR_INVALID, "bad head counts");
  const int G = n_q_heads / n_kv_heads;
  if (G > kMaxG) return noalloc_fail(NOSA_ERR_UNIMPLEMENTED, "group size %d > %d", G, kMaxG);
  if (k_sel < 1 || max_blocks < 1 || k_sel > max_blocks)
    return noalloc_fail(NOSA_ERR_INVALID, "need 1 <= k_sel <= max_blocks");
  const long long U = (long long)batch * n_kv_heads;
  if (U * max_blocks * kP >= (1ll << 31)) return noalloc_fail(NOSA_ERR_INVALID, "KV rows exceed 2^31");
  if (U * G > kNoAllocHeads)
    return noalloc_fail(NOSA_ERR_INVALID,
                        "batch x n_q_heads = %lld exceeds the %d query heads the fixed scratch holds", U * G,
                        kNoAllocHeads);
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) % 16 != 0)
    return noalloc_fail(NOSA_ERR_INVALID, "K/V base addresses must be 16-byte aligned");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  DeviceScratch* ds = nullptr;
  nosa_status s = device_scratch(dev, &ds);
  if (s != NOSA_OK) return s;

  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // The walk of a context over resident KV: k blocks, a tail position (never
  // valid here: there is no open tail) and the gap.  With the same grid the
  // CTAs cover the same blocks and write the same partials, so the output is
  // bit-identical to nosa_sparse_decode's on the same inputs.
  const int vpu = k_sel + 1 + kHitsGap;
  const int grid = attend_hits_grid((int)U, vpu, 2 * sms);
  const int nparts = attend_hits_parts((int)U, vpu, grid);
  if (U * nparts * G > kNoAllocRows)
    return noalloc_fail(NOSA_ERR_INVALID, "%lld partial rows exceed the fixed scratch of %d rows",
                        U * nparts * G, kNoAllocRows);

  DecodeMaps maps{};
  if ((s = encode_rows(&maps.k, k, (unsigned long long)U * max_blocks * kP)) != NOSA_OK) return s;
  if ((s = encode_rows(&maps.v, v, (unsigned long long)U * max_blocks * kP)) != NOSA_OK) return s;
  maps.tk = maps.k;  // there is no tail item
  maps.tv = maps.v;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the merge counters must start at zero (a call stopped by a timeout leaves
  // them behind); the error word is left alone: it accumulates until
  // nosa_noalloc_check_errors reads and clears it
  e = cudaMemsetAsync(ds->unit_done, 0, (size_t)U * sizeof(int), st);
  if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));

  DecodeArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.sel = sel;
  a.part_o = ds->part_o;
  a.part_ml = ds->part_ml;
  a.ds = ds->state;
  a.U = (int)U;
  a.Hq = n_q_heads;
  a.Hkv = n_kv_heads;
  a.G = G;
  a.k = k_sel;
  a.max_blocks = max_blocks;
  a.resident = 1;
  a.tail_split = 0;
  a.vpu = vpu;
  a.part_base = 0;
  a.nparts = nparts;
  a.hits_grid = grid;
  a.unit_done = ds->unit_done;
  a.out = static_cast<uint16_t*>(out);
  e = launch_attend_hits(a, maps, grid, st);
  if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
  return NOSA_OK;
}

NOSA_API nosa_status nosa_noalloc_check_errors(nosa_stream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  DeviceScratch* ds = nullptr;
  nosa_status s = device_scratch(dev, &ds);
  if (s != NOSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned bits = 0;
  e = cudaMemcpyAsync(&bits, &ds->state->error_bits, sizeof bits, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(&ds->state->error_bits, 0, sizeof bits, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return noalloc_fail(NOSA_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
  if (bits & ERR_TIMEOUT)
    return noalloc_fail(NOSA_ERR_TIMEOUT, "a bounded device wait ran out (bits 0x%x): outputs of that call are "
                        "incomplete", bits);
  if (bits)
    return noalloc_fail(NOSA_ERR_INVALID, "a selected block id was out of range (bits 0x%x): block 0 was read "
                        "in its place", bits);
  return NOSA_OK;
}

}  // extern "C"
