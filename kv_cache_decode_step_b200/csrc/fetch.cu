// fetch.cu -- cache planning (set difference + replacement mapping) and the
// zero-copy miss gather.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary):
//   §4     a set-difference kernel between old and new selections builds a
//          replacement mapping; only blocks unused by the current step are
//          swapped out, since GPU-resident blocks need not be contiguous; a
//          transfer kernel reads fine-grained 16 KiB blocks through unified
//          virtual addressing;
//   App. A per step, the cache-missed blocks move CPU -> GPU.
// Replacement order: free slots (lowest first), then resident blocks outside
// S(t) by (last step selected, block id) ascending.  The i-th miss (ascending
// block id) takes the i-th slot of that order.
#include "nosa_internal.cuh"

namespace nosa {

constexpr int kPlanWarps = 4;
constexpr unsigned kAll = 0xffffffffu;

// One warp per unit.  The unit's slot tables are staged in shared memory so
// the only dependent global round trips are sel -> block_slot.
__global__ void __launch_bounds__(kPlanWarps * 32) plan_kernel(PlanArgs a) {
  extern __shared__ int sm_plan[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kPlanWarps + warp;
  if (u >= a.U) return;
  int* sb = sm_plan + (size_t)warp * (2 * a.C + 2 * a.k);  // slot -> block
  int* lu = sb + a.C;                                       // slot -> last step selected
  int* smiss = lu + a.C;                                    // missed blocks, ascending
  int* ssrc = smiss + a.k;                                  // slots they will take

  const int t = a.ds->step;
  const int* sel = a.sel + (size_t)u * a.k;
  int* slot_block = a.slot_block + (size_t)u * a.C;
  int* last_used = a.last_used + (size_t)u * a.C;
  int* block_slot = a.block_slot + (size_t)u * a.max_blocks;
  int* items = a.items + (size_t)u * a.k;
  const unsigned lt = (1u << lane) - 1u;

  for (int c = lane; c < a.C; c += 32) {
    sb[c] = slot_block[c];
    lu[c] = last_used[c];
  }
  __syncwarp();

  // 1. hits refresh their stamp; misses are listed in ascending order
  int n_hit = 0, n_miss = 0;
  for (int i0 = 0; i0 < a.k; i0 += 32) {
    const int i = i0 + lane;
    const int bj = i < a.k ? sel[i] : -1;
    const bool valid = bj >= 0 && bj < a.max_blocks;
    const int slot = valid ? block_slot[bj] : -1;
    const bool hit = valid && slot >= 0 && slot < a.C;
    const bool miss = valid && !hit;
    const unsigned hm = __ballot_sync(kAll, hit), mm = __ballot_sync(kAll, miss);
    if (hit) {
      lu[slot] = t;
      last_used[slot] = t;
      items[n_hit + __popc(hm & lt)] = slot;
    }
    if (miss) smiss[n_miss + __popc(mm & lt)] = bj;
    n_hit += __popc(hm);
    n_miss += __popc(mm);
  }
  __syncwarp();

  // 2. free slots, lowest first
  int n_src = 0;
  for (int c0 = 0; c0 < a.C && n_src < n_miss; c0 += 32) {
    const int c = c0 + lane;
    const bool fr = c < a.C && sb[c] < 0;
    const unsigned fm = __ballot_sync(kAll, fr);
    const int pos = n_src + __popc(fm & lt);
    if (fr && pos < n_miss) ssrc[pos] = c;
    n_src += __popc(fm);
  }
  n_src = min(n_src, n_miss);
  __syncwarp();

  // 3. victims: resident, not selected now (stamp < t); least recent stamp,
  //    then lower block id, first.  Stamps are >= 0 for resident slots.
  bool failed = false;
  while (n_src < n_miss) {
    unsigned bhi = 0xffffffffu, blo = 0xffffffffu;
    for (int c = lane; c < a.C; c += 32) {
      const int bj = sb[c];
      const int st = lu[c];
      if (bj >= 0 && st < t) {
        const unsigned h = (unsigned)st, l = (unsigned)bj;
        if (h < bhi || (h == bhi && l < blo)) {
          bhi = h;
          blo = l;
        }
      }
    }
    const unsigned mhi = __reduce_min_sync(kAll, bhi);
    const unsigned mlo = __reduce_min_sync(kAll, bhi == mhi ? blo : 0xffffffffu);
    if (mhi == 0xffffffffu) {
      failed = true;
      break;
    }
    if (lane == 0) {
      const int victim_block = (int)mlo;
      const int vslot = block_slot[victim_block];
      ssrc[n_src] = vslot;
      block_slot[victim_block] = -1;
      sb[vslot] = -2;  // claimed; excluded from the search
      lu[vslot] = t;
    }
    ++n_src;
    __syncwarp();
  }
  if (failed) {
    if (lane == 0) atomicOr(&a.ds->error_bits, ERR_NOSLOT);
    n_miss = n_src;
  }

  // 4. install the misses and emit the gather list
  int base = 0;
  if (lane == 0 && n_miss > 0) base = atomicAdd(&a.ds->gather_count, n_miss);
  base = __shfl_sync(kAll, base, 0);
  int* fetch = a.fetch + (size_t)u * a.k;
  for (int i = lane; i < a.k; i += 32) {
    if (i < n_miss) {
      const int bj = smiss[i], c = ssrc[i];
      slot_block[c] = bj;
      block_slot[bj] = c;
      last_used[c] = t;
      items[n_hit + i] = c;
      fetch[i] = bj;
      a.glist[base + i] = make_int4(u, bj, c, 0);
    } else {
      fetch[i] = -1;
    }
  }
  if (lane == 0) {
    a.n_fetch[u] = n_miss;
    a.n_hit[u] = n_hit;
    a.n_items[u] = n_hit + n_miss;
    atomicAdd(&a.st->hits, (unsigned long long)n_hit);
    atomicAdd(&a.st->misses, (unsigned long long)n_miss);
    atomicAdd(&a.st->fetched_bytes, (unsigned long long)n_miss * 2ull * kBlockBytes);
    if (t > 0) atomicMax(&a.st->max_fetch, n_miss);
  }
}

// Register path for C <= 32 slots and k <= 32: lane s holds cache slot s and
// lane i holds the i-th selected block, so hits are found by matching the
// selection against the slot table with shuffles (no dependent global load)
// and the victim search is a pair of redux.sync minimums per victim.
__global__ void __launch_bounds__(kPlanWarps * 32) plan_reg_kernel(PlanArgs a) {
  __shared__ int ssrc_all[kPlanWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kPlanWarps + warp;
  if (u >= a.U) return;
  int* ssrc = ssrc_all[warp];
  const int t = a.ds->step;
  int* slot_block = a.slot_block + (size_t)u * a.C;
  int* last_used = a.last_used + (size_t)u * a.C;
  int* block_slot = a.block_slot + (size_t)u * a.max_blocks;
  int* items = a.items + (size_t)u * a.k;
  const unsigned lt = (1u << lane) - 1u;

  const bool has_slot = lane < a.C;
  int sb = has_slot ? slot_block[lane] : -3;
  const int lu = has_slot ? last_used[lane] : 0;
  const int bj = lane < a.k ? a.sel[(size_t)u * a.k + lane] : -1;
  const bool valid = bj >= 0 && bj < a.max_blocks;

  // 1. hits: the slot holding bj, if any (slots never hold a block twice)
  int slot = -1;
  for (int s2 = 0; s2 < a.C; ++s2) {
    const int v = __shfl_sync(kAll, sb, s2);
    if (valid && v == bj) slot = s2;
  }
  const bool hit = valid && slot >= 0;
  const bool miss = valid && slot < 0;
  const unsigned hm = __ballot_sync(kAll, hit), mm = __ballot_sync(kAll, miss);
  const int n_hit = __popc(hm), n_miss_all = __popc(mm);
  const unsigned hit_slots = __reduce_or_sync(kAll, hit ? (1u << slot) : 0u);
  const bool slot_hit = has_slot && ((hit_slots >> lane) & 1u);
  if (slot_hit) last_used[lane] = t;
  if (hit) items[__popc(hm & lt)] = slot;

  // 2. free slots, lowest first
  const unsigned fm = __ballot_sync(kAll, has_slot && sb < 0);
  if (has_slot && sb < 0) {
    const int r = __popc(fm & lt);
    if (r < n_miss_all) ssrc[r] = lane;
  }
  int n_src = min(__popc(fm), n_miss_all);

  // 3. victims: resident, not selected now, least recent stamp then lower id
  bool cand = has_slot && sb >= 0 && !slot_hit && lu < t;
  bool failed = false;
  while (n_src < n_miss_all) {
    const unsigned mhi = __reduce_min_sync(kAll, cand ? (unsigned)lu : 0xffffffffu);
    const unsigned mlo = __reduce_min_sync(kAll, (cand && (unsigned)lu == mhi) ? (unsigned)sb : 0xffffffffu);
    if (mhi == 0xffffffffu) {
      failed = true;
      break;
    }
    if (cand && (unsigned)lu == mhi && (unsigned)sb == mlo) {
      ssrc[n_src] = lane;
      block_slot[sb] = -1;
      cand = false;
    }
    ++n_src;
  }
  __syncwarp();
  int n_miss = n_miss_all;
  if (failed) {
    if (lane == 0) atomicOr(&a.ds->error_bits, ERR_NOSLOT);
    n_miss = n_src;
  }

  // 4. install the misses (ascending block order) and emit the gather list
  int base = 0;
  if (lane == 0 && n_miss > 0) base = atomicAdd(&a.ds->gather_count, n_miss);
  base = __shfl_sync(kAll, base, 0);
  const int mi = __popc(mm & lt);
  if (miss && mi < n_miss) {
    const int c = ssrc[mi];
    slot_block[c] = bj;
    last_used[c] = t;
    block_slot[bj] = c;
    items[n_hit + mi] = c;
    a.fetch[(size_t)u * a.k + mi] = bj;
    a.glist[base + mi] = make_int4(u, bj, c, 0);
  }
  for (int i = n_miss + lane; i < a.k; i += 32) a.fetch[(size_t)u * a.k + i] = -1;
  if (lane == 0) {
    a.n_fetch[u] = n_miss;
    a.n_hit[u] = n_hit;
    a.n_items[u] = n_hit + n_miss;
    atomicAdd(&a.st->hits, (unsigned long long)n_hit);
    atomicAdd(&a.st->misses, (unsigned long long)n_miss);
    atomicAdd(&a.st->fetched_bytes, (unsigned long long)n_miss * 2ull * kBlockBytes);
    if (t > 0) atomicMax(&a.st->max_fetch, n_miss);
  }
}

cudaError_t launch_plan(const PlanArgs& a, cudaStream_t st) {
  const int grid = (a.U + kPlanWarps - 1) / kPlanWarps;
  if (a.C <= 32 && a.k <= 32) {
    plan_reg_kernel<<<grid, kPlanWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)kPlanWarps * (2 * a.C + 2 * a.k) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  plan_kernel<<<grid, kPlanWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- gather
// Each CTA copies whole list entries: one entry is the K block and the V block
// of one (unit, block), 2 x 16 KiB, read from pinned host memory through its
// device address and written to the cache slot.  256 threads x 8 16-byte loads
// keep one entry (32 KiB) in flight per CTA.
constexpr int kGatherThreads = 256;

__device__ __forceinline__ uint4 ld_sys(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__global__ void __launch_bounds__(kGatherThreads) gather_kernel(GatherArgs a) {
  const int count = *a.count;
  // the most recently closed block may not have reached the host store yet:
  // it is read from its staging copy in HBM
  const int staged = a.stage_k ? a.ds->staged_block : -1;
  constexpr int kPer = kBlockBytes / 16 / kGatherThreads;  // 4 words of K (and of V) per thread
  for (int e = blockIdx.x; e < count; e += gridDim.x) {
    const int4 it = a.glist[e];
    if (it.x < 0 || it.x >= a.U || it.y < 0 || it.y >= a.max_blocks || it.z < 0 || it.z >= a.C) {
      if (threadIdx.x == 0) atomicOr(&a.ds->error_bits, ERR_RANGE);
      continue;
    }
    const size_t src = ((size_t)it.x * a.max_blocks + it.y) * (kBlockBytes / 16);
    const size_t dst = ((size_t)it.x * a.C + it.z) * (kBlockBytes / 16);
    const bool from_stage = it.y == staged;
    const size_t s0 = from_stage ? (size_t)it.x * (kBlockBytes / 16) : src;
    const uint4* sk = reinterpret_cast<const uint4*>(from_stage ? a.stage_k : a.hk) + s0;
    const uint4* sv = reinterpret_cast<const uint4*>(from_stage ? a.stage_v : a.hv) + s0;
    uint4* dk = reinterpret_cast<uint4*>(a.ck) + dst;
    uint4* dv = reinterpret_cast<uint4*>(a.cv) + dst;
    uint4 rk[kPer], rv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      rk[i] = ld_sys(sk + threadIdx.x + i * kGatherThreads);
      rv[i] = ld_sys(sv + threadIdx.x + i * kGatherThreads);
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      dk[threadIdx.x + i * kGatherThreads] = rk[i];
      dv[threadIdx.x + i * kGatherThreads] = rv[i];
    }
  }
}

// The gather is launched with the device's highest CTA priority so that its
// few CTAs are dispatched ahead of the attention CTAs that run concurrently
// on the compute stream; otherwise the PCIe transfer starts only once
// attention has drained.
cudaError_t launch_gather(const GatherArgs& a, int grid, cudaStream_t st) {
  int least = 0, greatest = 0;
  cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGatherThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributePriority;
  attr[0].val.priority = greatest;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gather_kernel, a);
}

}  // namespace nosa
