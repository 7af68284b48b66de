// rows.cu -- zero-copy row gather at a chosen granularity.
//
// The decode step moves each missed KV block as one 16 KiB row of K and one of
// V (NOSA: Native and Offloadable Sparse Attention, paperlayer summary, §4:
// fine-grained 16 KiB transfers through unified virtual addressing).  The
// same summary (§3.2) contrasts block-wise with element-wise transfer, where
// each selected token's key and value rows (256 bytes each at d = 128, bf16)
// cross PCIe separately.  nosa_gather_rows moves rows of any power-of-two size
// from 16 bytes to 64 KiB, so one kernel measures both granularities on the
// same miss volume.
#include <cstdarg>
#include <cstdio>

#include "../../include/nosa.h"
#include "nosa_internal.cuh"

namespace nosa {
namespace {

constexpr int kRowsThreads = 256;
constexpr int kRowsUnroll = 4;  // independent 16-byte loads in flight per thread

struct RowsArgs {
  const uint4* src;
  uint4* dst;
  const int64_t* src_idx;
  const int64_t* dst_idx;   // NULL: row i goes to row i
  long long src_rows, dst_rows;
  long long total;          // 16-byte chunks to move = n << log_cpr
  int log_cpr;              // log2(chunks per row)
  uint32_t* flags;          // NULL or bit 0 set on an out-of-range index
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Chunk c of the flattened copy is chunk (c mod cpr) of row (c / cpr).  A warp
// covers 32 consecutive chunks (512 bytes), so a row of 256 bytes or more is
// read with whole-warp coalesced accesses; each thread keeps kRowsUnroll
// loads, one grid stride apart, in flight before storing.
__global__ void __launch_bounds__(kRowsThreads) gather_rows_kernel(RowsArgs a) {
  const long long stride = (long long)gridDim.x * kRowsThreads;
  const long long mask = (1ll << a.log_cpr) - 1;
  for (long long c0 = (long long)blockIdx.x * kRowsThreads + threadIdx.x; c0 < a.total;
       c0 += kRowsUnroll * stride) {
    uint4 r[kRowsUnroll];
    long long d[kRowsUnroll];
#pragma unroll
    for (int j = 0; j < kRowsUnroll; ++j) {
      const long long c = c0 + j * stride;
      d[j] = -1;
      if (c < a.total) {
        const long long row = c >> a.log_cpr;
        const long long s = __ldg(a.src_idx + row);
        const long long t = a.dst_idx ? __ldg(a.dst_idx + row) : row;
        if (s < 0 || s >= a.src_rows || t < 0 || t >= a.dst_rows) {
          if (a.flags) atomicOr(a.flags, 1u);
        } else {
          r[j] = ld_stream(a.src + ((s << a.log_cpr) | (c & mask)));
          d[j] = (t << a.log_cpr) | (c & mask);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kRowsUnroll; ++j)
      if (d[j] >= 0) a.dst[d[j]] = r[j];
  }
}

// ---------------------------------------------------------------- bulk copies
// The same row gather through the TMA unit: each row (or 16 KiB piece of a
// longer row) is one cp.async.bulk global -> shared load, completing on an
// mbarrier, then one cp.async.bulk shared -> global store.  Every warp is an
// independent copier whose lane 0 keeps up to kBulkSlots pieces in flight in
// its own ring of shared-memory slots.  The copy engine of the TMA unit issues
// its own memory requests, so the PCIe read requests are not shaped by 16-byte
// SM loads.
constexpr int kBulkThreads = 128;
constexpr int kBulkWarps = kBulkThreads / 32;
constexpr int kBulkSlots = 8;                  // most pieces in flight per warp
constexpr int kBulkRingBytes = 48 * 1024;      // shared memory per warp
constexpr int kBulkSmemBytes = 1024 + kBulkWarps * kBulkRingBytes;
constexpr int kBulkPieceMax = 16384;
constexpr uint64_t kBulkWaitNs = 1000000000ull;


// a.total counts pieces here, log_piece = log2(piece bytes), a.log_cpr =
// log2(pieces per row); nslots = min(kBulkSlots, kBulkRingBytes / piece).
__global__ void __launch_bounds__(kBulkThreads) gather_rows_bulk_kernel(RowsArgs a, int log_piece, int nslots) {
  extern __shared__ __align__(1024) unsigned char bulk_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane != 0) return;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bulk_smem) + warp * kBulkSlots;
  unsigned char* ring = bulk_smem + 1024 + warp * kBulkRingBytes;
  const uint32_t piece = 1u << log_piece;
  for (int s = 0; s < nslots; ++s) mbar_init(&bars[s], 1);
  fence_mbar_init();
  const long long agents = (long long)gridDim.x * kBulkWarps;
  const long long mask = (1ll << a.log_cpr) - 1;
  const unsigned char* src = reinterpret_cast<const unsigned char*>(a.src);
  unsigned char* dst = reinterpret_cast<unsigned char*>(a.dst);
  long long next = (long long)blockIdx.x * kBulkWarps + warp;  // next piece this warp considers
  long long dst_off[kBulkSlots];
  int head = 0, tail = 0;  // pieces loaded (issued), pieces stored
  // issue the next in-range piece into slot head % nslots; false when none is left
  auto issue = [&]() -> bool {
    while (next < a.total) {
      const long long c = next;
      next += agents;
      const long long row = c >> a.log_cpr;
      const long long s = __ldg(a.src_idx + row);
      const long long t = a.dst_idx ? __ldg(a.dst_idx + row) : row;
      if (s < 0 || s >= a.src_rows || t < 0 || t >= a.dst_rows) {
        if (a.flags) atomicOr(a.flags, 1u);
        continue;
      }
      const int slot = head % nslots;
      const long long off = (c & mask) << log_piece;
      dst_off[slot] = ((t << a.log_cpr) << log_piece) + off;
      mbar_arrive_expect_tx(&bars[slot], piece);
      bulk_load(ring + (size_t)slot * piece, src + ((s << a.log_cpr) << log_piece) + off, piece, &bars[slot]);
      ++head;
      return true;
    }
    return false;
  };
  while (head < nslots && issue()) {
  }
  while (tail < head) {
    const int slot = tail % nslots;
    if (!mbar_wait_bounded(&bars[slot], (uint32_t)((tail / nslots) & 1), kBulkWaitNs)) {
      // record, give the other loads in flight a bounded chance to land, stop
      if (a.flags) atomicOr(a.flags, 2u);
      for (int g = tail + 1; g < head; ++g)
        (void)mbar_wait_bounded(&bars[g % nslots], (uint32_t)((g / nslots) & 1), kBulkWaitNs);
      break;
    }
    bulk_store(dst + dst_off[slot], ring + (size_t)slot * piece, piece);
    bulk_commit();
    ++tail;
    // the slot of the piece just stored is reloaded once the store has read it
    bulk_wait_read_all();
    issue();
  }
  bulk_wait_all();
}

nosa_status rows_fail(nosa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  record_error(buf);
  return s;
}

}  // namespace
}  // namespace nosa

namespace nosa {
namespace {

// Validation and argument set-up shared by both gathers; *grid is the CTA
// count asked for (0: a quarter of the SMs).
nosa_status rows_setup(const void* src, int64_t src_rows, void* dst, int64_t dst_rows, int32_t row_bytes,
                       const int64_t* src_idx, const int64_t* dst_idx, int32_t n, int32_t ctas, uint32_t* flags,
                       RowsArgs* a, int* grid) {
  if (n < 0) return rows_fail(NOSA_ERR_INVALID, "n = %d < 0", n);
  if (row_bytes < 16 || row_bytes > 65536 || (row_bytes & (row_bytes - 1)) != 0)
    return rows_fail(NOSA_ERR_INVALID, "row_bytes = %d is not a power of two in [16, 65536]", row_bytes);
  if (ctas < 0 || ctas > 65535) return rows_fail(NOSA_ERR_INVALID, "ctas = %d outside [0, 65535]", ctas);
  if (src_rows < 0 || dst_rows < 0) return rows_fail(NOSA_ERR_INVALID, "negative row counts");
  *grid = 0;
  if (n == 0) return NOSA_OK;
  if (!src || !dst || !src_idx) return rows_fail(NOSA_ERR_INVALID, "NULL argument");
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % 16 != 0)
    return rows_fail(NOSA_ERR_INVALID, "src and dst must be 16-byte aligned");
  // Only memory the device can address is accepted: a pageable host pointer
  // is rejected here rather than handed to the kernel.
  void* src_dev = nullptr;
  void* dst_dev = nullptr;
  void* idx_dev = nullptr;
  if (pointer_kind(src, &src_dev) == 0)
    return rows_fail(NOSA_ERR_INVALID, "src is neither device memory nor pinned host memory");
  if (pointer_kind(dst, &dst_dev) != 1) return rows_fail(NOSA_ERR_INVALID, "dst must be device memory");
  if (pointer_kind(src_idx, &idx_dev) != 1 || (dst_idx && pointer_kind(dst_idx, &idx_dev) != 1))
    return rows_fail(NOSA_ERR_INVALID, "index arrays must be device memory");
  if (flags && pointer_kind(flags, &idx_dev) != 1) return rows_fail(NOSA_ERR_INVALID, "flags must be device memory");
  int log_cpr = 0;
  while ((16 << log_cpr) < row_bytes) ++log_cpr;
  if (src_rows > (1ll << 59 >> log_cpr) || dst_rows > (1ll << 59 >> log_cpr))
    return rows_fail(NOSA_ERR_INVALID, "row counts too large");
  int g = ctas;
  if (g == 0) {
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return rows_fail(NOSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    g = (sms + 3) / 4;
  }
  *a = RowsArgs{};
  a->src = static_cast<const uint4*>(src_dev);
  a->dst = static_cast<uint4*>(dst_dev);
  a->src_idx = src_idx;
  a->dst_idx = dst_idx;
  a->src_rows = src_rows;
  a->dst_rows = dst_rows;
  a->total = (long long)n << log_cpr;
  a->log_cpr = log_cpr;
  a->flags = flags;
  *grid = g;
  return NOSA_OK;
}

}  // namespace
}  // namespace nosa

using namespace nosa;

extern "C" {

NOSA_API nosa_status nosa_gather_rows(const void* src, int64_t src_rows, void* dst, int64_t dst_rows,
                                      int32_t row_bytes, const int64_t* src_idx, const int64_t* dst_idx,
                                      int32_t n, int32_t ctas, uint32_t* flags, nosa_stream_t stream) {
  RowsArgs a;
  int grid = 0;
  nosa_status s = rows_setup(src, src_rows, dst, dst_rows, row_bytes, src_idx, dst_idx, n, ctas, flags, &a, &grid);
  if (s != NOSA_OK || grid == 0) return s;
  const long long need = (a.total + kRowsThreads * kRowsUnroll - 1) / (kRowsThreads * kRowsUnroll);
  if (grid > need) grid = (int)need;
  gather_rows_kernel<<<grid, kRowsThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return rows_fail(NOSA_ERR_CUDA, "gather launch: %s", cudaGetErrorString(e));
  return NOSA_OK;
}

NOSA_API nosa_status nosa_gather_rows_bulk(const void* src, int64_t src_rows, void* dst, int64_t dst_rows,
                                           int32_t row_bytes, const int64_t* src_idx, const int64_t* dst_idx,
                                           int32_t n, int32_t ctas, uint32_t* flags, nosa_stream_t stream) {
  RowsArgs a;
  int grid = 0;
  nosa_status s = rows_setup(src, src_rows, dst, dst_rows, row_bytes, src_idx, dst_idx, n, ctas, flags, &a, &grid);
  if (s != NOSA_OK || grid == 0) return s;
  // pieces of at most 16 KiB: a.total and a.log_cpr count pieces, not 16-byte words
  int log_piece = 4;
  while ((1 << log_piece) < row_bytes && (2 << log_piece) <= kBulkPieceMax) ++log_piece;
  int log_rb = 4;
  while ((1 << log_rb) < row_bytes) ++log_rb;
  a.log_cpr = log_rb - log_piece;
  a.total = (long long)n << a.log_cpr;
  int nslots = kBulkRingBytes >> log_piece;
  if (nslots > kBulkSlots) nslots = kBulkSlots;
  const long long need = (a.total + kBulkWarps - 1) / kBulkWarps;
  if (grid > need) grid = (int)need;
  static bool configured = false;  // per process; the attribute is per device function
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gather_rows_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kBulkSmemBytes);
    if (e != cudaSuccess) return rows_fail(NOSA_ERR_CUDA, "bulk gather configuration: %s", cudaGetErrorString(e));
    configured = true;
  }
  gather_rows_bulk_kernel<<<grid, kBulkThreads, kBulkSmemBytes, reinterpret_cast<cudaStream_t>(stream)>>>(
      a, log_piece, nslots);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return rows_fail(NOSA_ERR_CUDA, "bulk gather launch: %s", cudaGetErrorString(e));
  return NOSA_OK;
}

}  // extern "C"
