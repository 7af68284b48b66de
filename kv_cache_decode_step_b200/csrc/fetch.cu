// fetch.cu -- cache planning (set difference + replacement mapping) and the
// zero-copy miss gather.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary):
//   §4     the old and new selections are compared by a dedicated kernel
//          that decides which cached blocks give up their slots; a block
//          the step still needs keeps its slot, and slots need not be
//          contiguous; a transfer kernel reads 16 KiB blocks from host memory
//          through unified virtual addressing;
//   App. A per step, the cache-missed blocks move CPU -> GPU.
// Replacement order: free slots (lowest first), then resident blocks outside
// S(t) by (last step selected, block id) ascending.  The i-th miss (ascending
// block id) takes the i-th slot of that order.
#include "plan_dev.cuh"

namespace nosa {

constexpr int kPlanWarps = 4;

// One warp per unit; dynamic shared memory of kPlanWarps * (2C + 2k) ints.
__global__ void __launch_bounds__(kPlanWarps * 32) plan_kernel(PlanArgs a) {
  extern __shared__ int sm_plan[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kPlanWarps + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.ds->gather_next = 0;  // see prepare_kernel
  if (u >= a.U) return;
  plan_unit_smem(a, u, lane, sm_plan + (size_t)warp * (2 * a.C + 2 * a.k), a.sel + (size_t)u * a.k,
                 a.block_slot + (size_t)u * a.max_blocks, false);
}

// Register path for C <= 32 slots and k <= 32.
__global__ void __launch_bounds__(kPlanWarps * 32) plan_reg_kernel(PlanArgs a) {
  __shared__ int ssrc_all[kPlanWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kPlanWarps + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.ds->gather_next = 0;  // see prepare_kernel
  if (u >= a.U) return;
  plan_unit_reg(a, u, lane, ssrc_all[warp], a.sel + (size_t)u * a.k, a.slot_block + (size_t)u * a.C,
                a.last_used + (size_t)u * a.C);
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
