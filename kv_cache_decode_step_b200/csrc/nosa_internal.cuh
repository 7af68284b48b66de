// nosa_internal.cuh -- device-side state, kernel parameter blocks and inline PTX
// shared by the kernels of libnosa.so.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nosa {

constexpr int kD = 128;     // head dim
constexpr int kP = 64;      // tokens per block
constexpr int kQ = 16;      // tokens per sub-block
constexpr int kR = kP / kQ; // sub-blocks per block
constexpr int kMaxG = 8;    // query heads per KV head (mma N = 8)
constexpr int kRowU4 = kD * 2 / 16;  // 16-byte words per token row (16)
constexpr int kBlockBytes = kP * kD * 2;  // 16 KiB: one block of K (or of V)

enum : unsigned {
  ERR_TIMEOUT = 1u,
  ERR_CAPACITY = 2u,
  ERR_NOSLOT = 4u,
  ERR_RANGE = 8u,
};

// Per-step quantities live on the device so that a captured step replays
// correctly.  Written only by single-thread kernels or by one elected thread
// whose writes no other thread of the same launch reads.
struct DevState {
  int step;            // selections completed (t of the step in flight)
  int n_closed;        // closed blocks per unit
  int n_last_select;   // n_closed seen by the previous selection
  int tail_len;        // tokens in the open tail at the start of the step
  int tail_len_step;   // tail length during the step (tail_len + appended)
  int gather_count;    // entries in the gather list of the current step
  unsigned error_bits;
  int staged_block;    // closed block whose K/V sit in the staging buffer, -1 none
  int wt_block;        // staged block not yet written through to the store, -1 none
  int wt_done;         // CTAs of the write-through launch that have finished
  int gather_next;     // next gather-list entry to claim (reset by the kernel that plans the step)
  int pad;
};

struct DevStats {
  unsigned long long steps, selected, hits, misses, fetched_bytes, overlap_sum, overlap_terms;
  int min_overlap, max_fetch;
};

// ------------------------------------------------------------------ PTX

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialization attribute may have its CTAs placed while the kernel
// before it on the stream is still running; grid_dep_wait() returns once that
// kernel has completed and its writes are visible, so everything a kernel
// reads from its predecessor comes after it.  Launched without the attribute,
// the wait returns at once.  grid_dep_launch() lets such a dependent be placed
// as soon as every CTA of this grid has issued it (or exited); the dependent's
// CTAs then wait on the SMs instead of being launched after the completion.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of an mbarrier, giving up after limit_ns of
// globaltimer (or a hard iteration cap).  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < (1u << 26); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 127u) == 0 && global_timer_ns() - t0 > limit_ns) return false;
  }
  return false;
}

// 2-D tiled TMA load of one box into this CTA's shared memory only, completing
// on an mbarrier.  x is the innermost coordinate (elements), y the row.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// The same load with an L2 cache policy (see l2_evict_first_policy).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// An L2 policy that makes the lines a load brings in the first to go: for
// data read once per step (the selected K/V), so that it does not push out
// data reused across steps (the pooled keys) first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Bulk prefetch of global memory into L2 (no data reaches the SM).  Address
// 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
               : "memory");
}

// Untiled bulk copy global -> this CTA's shared memory, completing on an
// mbarrier.  Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Untiled bulk copy shared -> global in this thread's bulk async-group,
// committed; wait_read: this thread's groups have read their shared memory;
// wait_all: and completed.
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(gdst)),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Plain arrival on an mbarrier (no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D(16x8, fp32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8x8 b16 matrix held one row-pair per lane (row lane/4, columns
// 2*(lane%4) and +1) across the warp.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 4-byte asynchronous copy global -> shared (completes at cp_async_wait_all).
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// 8- and 16-byte asynchronous copies global -> shared, in this thread's
// current group; commit closes the group, wait_group<N> waits until at most N
// of this thread's committed groups are pending.
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ double bf16_lo_to_f64(uint32_t w) { return (double)__uint_as_float(w << 16); }
__device__ __forceinline__ double bf16_hi_to_f64(uint32_t w) {
  return (double)__uint_as_float(w & 0xFFFF0000u);
}
// The upper bf16 of w times 2^-896, exactly, without a conversion
// instruction: its sign, 8 exponent bits and 7 fraction bits placed in the
// fp64 high word so that the 8-bit exponent sits in the low bits of the
// 11-bit field (3 bits lower than bf16 -> fp32 places it).  The fp64 bias
// (1023) exceeds bf16's (127) by 896, so a normal bf16 keeps its fraction and
// loses 2^896 of scale, and a zero or subnormal bf16 (exponent 0) becomes the
// fp64 zero or subnormal of the same fraction, again 2^896 smaller.  A product
// with an operand scaled up by 2^896 is therefore the same real number as the
// unscaled product and rounds identically.  Finite inputs only.
constexpr double kBf16PlaceScale = 0x1p896;
__device__ __forceinline__ double bf16_hi_placed_f64(uint32_t w) {
  const uint32_t hi = ((w & 0x7FFF0000u) >> 3) | (w & 0x80000000u);
  return __hiloint2double((int)hi, 0);
}

// fp64 -> bf16 with round-to-nearest-even, by integer rounding of the fp64
// significand to the bf16 grid (8 significant bits; spacing 2^-133 below
// 2^-126), overflow to infinity.
__device__ __forceinline__ uint32_t f64_to_bf16_bits(double x) {
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  const uint32_t sign = static_cast<uint32_t>(u >> 48) & 0x8000u;
  const unsigned long long mag = u & 0x7FFFFFFFFFFFFFFFull;
  if (mag > 0x7FF0000000000000ull) return 0x7FC0u;
  if (mag == 0x7FF0000000000000ull) return sign | 0x7F80u;
  const int e = static_cast<int>(mag >> 52);
  if (e == 0) return sign;  // fp64 subnormal: far below half the bf16 spacing
  const int E = e - 1023;
  const unsigned long long m = (mag & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  const int Eq = (E < -126 ? -126 : E) - 7;  // exponent of the bf16 grid spacing
  const int shift = Eq - (E - 52);           // low significand bits to drop (>= 45)
  if (shift >= 54) return sign;              // value < half a grid step
  unsigned long long q = m >> shift;
  const unsigned long long rem = m & ((1ull << shift) - 1);
  const unsigned long long half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (q & 1ull))) ++q;
  int bits = ((Eq + 7 + 126) << 7) + static_cast<int>(q);
  if (bits >= 0x7F80) bits = 0x7F80;
  return sign | static_cast<uint32_t>(bits);
}

// End of a step: the selection just made saw n_closed blocks; a full tail
// becomes a closed block; the step counter advances.  Run by one thread after
// every other kernel of the step has finished reading the state.
__device__ __forceinline__ void advance_step(DevState* ds, DevStats* st) {
  ds->n_last_select = ds->n_closed;
  const int tl = ds->tail_len_step;
  if (tl >= kP) {
    ds->n_closed += 1;
    ds->tail_len = 0;
  } else {
    ds->tail_len = tl;
  }
  ds->tail_len_step = ds->tail_len;
  ds->gather_count = 0;
  ds->step += 1;
  st->steps += 1;
}

// ------------------------------------------------------------------ launches
// Each returns the launch error (cudaSuccess if queued).

// Pooled keys of sub-blocks [s_begin, s_end) of every unit.
// src: bf16 [U, src_unit_tokens, d] (device or mapped host); kbar: bf16
// [U, kbar_unit_rows, d].
cudaError_t launch_pool(const uint16_t* src, size_t src_unit_tokens, int U, int s_begin, int s_end,
                        uint16_t* kbar, int kbar_unit_rows, cudaStream_t st);

struct ScoreArgs {
  const uint16_t* q;        // [B, Hq, d]; device memory, or mapped pinned host memory when q_copy is set
  uint16_t* q_copy;         // null, or [B, Hq, d] device: the fused kernel reads each unit's queries once
                            // (staged in shared memory) and leaves a device copy here for the attention
  const uint16_t* kbar;     // [U, max_blocks*R, d]
  double* scores;           // [U, max_blocks]
  DevState* ds;
  int U, Hq, Hkv, G, max_blocks;
  int placed_widen;         // 1: half of the keys widened by bit placement (same results)
};
cudaError_t launch_score(const ScoreArgs& a, cudaStream_t st);

struct SelectArgs {
  const float* agnostic;    // [U, max_blocks]
  const double* scores;     // [U, max_blocks]
  int* ge;                  // [U, k_e] state, ascending
  int* prev;                // [U, k] state S(t-1), ascending, -1 pad
  int* sel;                 // [U, k] output
  DevState* ds;
  DevStats* st;
  int U, max_blocks, k_q, k_e, k, c_max, words;
  int sink, window;         // forced blocks, counted inside k_e
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t st);

struct PlanArgs {
  const int* sel;           // [U, k]
  int* fetch;               // [U, k] output, -1 pad
  int* n_fetch;             // [U] output
  int* slot_block;          // [U, C]
  int* last_used;           // [U, C]
  int* block_slot;          // [U, max_blocks]
  int* items;               // [U, k] cache slots: hits then misses
  int* n_hit;               // [U]
  int* n_items;             // [U]
  int4* glist;              // [U*k] gather list (unit, block, slot)
  DevState* ds;
  DevStats* st;
  int U, k, C, max_blocks;
};
cudaError_t launch_plan(const PlanArgs& a, cudaStream_t st);

// Score, selection and plan of each unit in one launch (one CTA per unit);
// for max_blocks <= kPrepareMaxBlocks.  Needs gather_count = 0 on entry,
// which every step's end leaves behind.
constexpr int kPrepareMaxBlocks = 512;
struct PrepareArgs {
  ScoreArgs sc;
  SelectArgs se;
  PlanArgs pl;              // with KV resident only fetch / n_fetch are used
  int offloaded;
  int nwarps;               // warps per CTA (4..16): more when there are few units
  int plan_ints;            // set by the launcher
  // KV in HBM: while warp 0 selects, warp 1 asks L2 for the blocks that the
  // hits-pass CTAs starting in this unit load first (warm_blocks each), as
  // S(t-1) places them (S(t) keeps at least m of its blocks).  Null: off.
  const uint16_t* warm_k;   // resident K / V [U, max_blocks*P, d]
  const uint16_t* warm_v;
  int warm_blocks, hits_vpu, hits_grid;
};
bool prepare_supported(int max_blocks);
cudaError_t launch_prepare(const PrepareArgs& a, cudaStream_t st);
// Selection and plan in one launch (one warp per unit), after score_kernel;
// for max_blocks <= 1024.  Same results as launch_select then launch_plan.
// pdl: launched as a programmatic dependent of the kernel before it on `st`
// (the score kernel, which lets its dependents be placed early).
bool select_plan_supported(int max_blocks);
cudaError_t launch_select_plan(const SelectArgs& se, const PlanArgs& pl, int offloaded, cudaStream_t st,
                               bool pdl = false);

struct GatherArgs {
  const uint16_t* hk;       // host K (device-addressable), [U, max_blocks*P, d]
  const uint16_t* hv;
  uint16_t* ck;             // cache K [U, C, P, d]
  uint16_t* cv;
  const int4* glist;
  const int* count;         // entries to copy (device)
  const uint16_t* stage_k;  // [U, P, d] last closed block (null: nothing staged)
  const uint16_t* stage_v;
  DevState* ds;
  int U, C, max_blocks;
};
cudaError_t launch_gather(const GatherArgs& a, int grid, cudaStream_t st);

struct DecodeArgs {
  const uint16_t* q;        // [B, Hq, d]
  const int* sel;           // resident: [U, k] block ids
  const int* items;         // offloaded: [U, k] cache slots, hits first
  const int* n_hit;         // [U]
  const int* n_items;       // [U]
  float* part_o;            // [U, nparts, G, d]
  float2* part_ml;          // [U, nparts, G]
  DevState* ds;
  int U, Hq, Hkv, G, k, max_blocks, C;
  int resident;             // 1: sel indexes the resident KV
  int tail_split;           // 1: each unit's open tail is attended in the hits pass
  int vpu;                  // hits-pass positions per unit: k + tail_split + the gap (kHitsGap)
  int part_base, nparts;    // hits pass writes slots part_base + segment; nparts per unit
  int miss_base;            // slot of a unit's first fetched-block partial
  int hits_grid;            // CTAs of the hits pass (fixes each unit's segment count)
  int kv_evict_first;       // 1: the hits pass loads K/V with the L2 evict-first policy
  int* unit_done;           // [U] partials written this step; completing one merges the unit
  uint16_t* out;            // [B, Hq, d]
  int* done_ctr;            // non-null: units merged; the last merge ends the step (advance_step)
  DevStats* st;
};
struct DecodeMaps {
  CUtensorMap k, v;         // main K/V: resident KV or the cache, rows of 128 bf16
  CUtensorMap tk, tv;       // open tail blocks
};
// Hits pass (persistent, `grid` CTAs, which must equal a.hits_grid); partials,
// and with unit_done the output.
// producer_warp: the variant with a producer warp of its own (same results).
cudaError_t launch_attend_hits(const DecodeArgs& a, const DecodeMaps& m, int grid, cudaStream_t st,
                               int stages = 3, bool producer_warp = true);
// The hits-pass grid for a requested CTA count (at most one CTA per position).
int attend_hits_grid(int U, int vpu, int want);
// Partial slots per unit the hits pass writes for this shape and requested grid.
int attend_hits_parts(int U, int vpu, int want);
// Empty positions after each unit's blocks (and tail) in the hits pass walk.
constexpr int kHitsGap = 3;
// Kernel attributes (shared memory) of the attention kernels; once per device.
cudaError_t configure_decode();
cudaError_t configure_gather_attend();

// The miss gather fused with the attention of each fetched block: copies every
// entry of the gather list into its cache slot and, from shared memory, writes
// the block's partial (slot miss_base + entry.w of its unit), merging the unit
// when that completes its partials.  Highest CTA priority.
struct GatherAttendArgs {
  GatherArgs g;
  DecodeArgs d;
};
cudaError_t launch_gather_attend(const GatherAttendArgs& a, int grid, cudaStream_t st, bool pdl = false);

// Launch of `kernel` on `st`; with pdl, as a programmatic dependent of the
// kernel before it on the stream (the kernel must call grid_dep_wait() before
// it reads anything that kernel writes); priority: CTA priority, or 0.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                      int priority, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (priority != 0) {
    attr[n].id = cudaLaunchAttributePriority;
    attr[n].val.priority = priority;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Named barriers (bar.sync / bar.arrive over `count` threads, whole warps).
__device__ __forceinline__ void bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier over `count` threads that also ORs a predicate across them.
__device__ __forceinline__ bool bar_red_or(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

struct AppendArgs {
  const uint16_t* k_new;    // [B, Hkv, d]
  const uint16_t* v_new;
  const float* a_close;     // [U] or null
  uint16_t* tail_k;         // [U, P, d]
  uint16_t* tail_v;
  float* a_pending;         // [U]
  DevState* ds;
  int U, max_blocks;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t st);

struct CloseArgs {
  const uint16_t* tail_k;
  const uint16_t* tail_v;
  const float* a_pending;
  uint16_t* kbar;           // [U, max_blocks*R, d]
  float* agnostic;          // [U, max_blocks]
  uint16_t* kv_k;           // attached K (host mapped or device) [U, max_blocks*P, d]
  uint16_t* kv_v;
  uint16_t* stage_k;        // [U, P, d] or null: the closed block goes to the store directly
  uint16_t* stage_v;
  DevState* ds;
  int U, max_blocks;
};
cudaError_t launch_close(const CloseArgs& a, cudaStream_t st);

struct WriteThroughArgs {
  const uint16_t* stage_k;  // [U, P, d]
  const uint16_t* stage_v;
  uint16_t* kv_k;           // attached K in pinned host memory (device address)
  uint16_t* kv_v;
  DevState* ds;
  int U, max_blocks;
};
// Low CTA priority; returns at once when no staged block is pending.
cudaError_t launch_write_through(const WriteThroughArgs& a, int grid, cudaStream_t st);

cudaError_t launch_advance(DevState* ds, DevStats* st, cudaStream_t s);
// Sets the calling thread's nosa_last_error() message.
void record_error(const char* msg);

// Classify a pointer: 1 device (or managed) memory, 2 pinned or registered host
// memory, whose device address is stored in *dev_ptr; 0 anything else.
int pointer_kind(const void* p, void** dev_ptr);
cudaError_t launch_init_state(DevState* ds, int n_closed, int tail_len, int step, int n_last_select,
                              cudaStream_t s);
cudaError_t launch_reset_stats(DevStats* st, cudaStream_t s);
cudaError_t launch_wait_flag(const volatile int* flag, DevState* ds, long long timeout_ns, cudaStream_t s);

}  // namespace nosa
