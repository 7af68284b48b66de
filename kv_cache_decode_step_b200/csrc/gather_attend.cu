// gather_attend.cu -- the miss gather fused with the attention of each
// fetched block.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary): §4 (a
// transfer kernel moves fine-grained 16 KiB blocks from host memory through
// unified virtual addressing) and App. A (the missed blocks move CPU -> GPU,
// then attention runs over the GPU-resident blocks).  Here a fetched block is
// attended while it is still on chip: the copy that lands it in its cache
// slot also writes it into shared memory, and the block's partial is computed
// from there, so no pass over the fetched blocks has to wait for the whole
// transfer or read them back from HBM.
//
// A CTA is two roles over a ring of two 32 KiB stages:
//   8 copy warps    16-byte zero-copy loads of the entry's K and V from pinned
//                   host memory (or from the staging copy of a block closed by
//                   the previous step), stored to the cache slot and, in the
//                   tile layout of attend_dev.cuh, to the stage;
//   4 attention     the block's attention on the stage, its partial, and the
//     warps         unit's merge when that partial completes the unit.
// PCIe throughput follows the number of warps with loads in flight, hence the
// larger copy role.
// The roles hand stages over with named barriers (FULL: copy -> attention,
// EMPTY: attention -> copy), the entry riding with the stage, so every
// barrier phase has all its arrivals.  Nothing waits on another CTA.  The
// kernel may be launched as a programmatic dependent of the planning kernel:
// its CTAs are then placed while the plan finishes and read the plan only
// after it has completed.
#include "attend_dev.cuh"

namespace nosa {

constexpr int kGaCopy = 256;              // warps 0-7 copy
constexpr int kGaRole = 128;              // warps 8-11 attend
constexpr int kGaThreads = kGaCopy + kGaRole;
constexpr int kGaStages = 2;
constexpr int kGaStageBytes = 2 * kBlockBytes;
constexpr int kGaWsBytes = (4 * kMaxG * kD + 2 * 4 * kMaxG) * 4;
constexpr int kGaSmemBytes = kGaStages * kGaStageBytes + kGaWsBytes + 32;  // + flag, count, staged, 2 entries
constexpr int kBarFull = 1;               // ids 1, 2: stage s full
constexpr int kBarEmpty = 3;              // ids 3, 4: stage s free
constexpr int kBarAttn = 5;               // the attention warps alone
constexpr int kBarCopy = 6;               // the copy warps alone
constexpr int kGaPer = kBlockBytes / 16 / kGaCopy;  // 16-byte words of K (and of V) per copy thread

__device__ __forceinline__ uint4 ld_host(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ bool entry_valid(const GatherArgs& g, const DecodeArgs& a, const int4& it) {
  return it.x >= 0 && it.x < g.U && it.y >= 0 && it.y < g.max_blocks && it.z >= 0 && it.z < g.C && it.w >= 0 &&
         it.w < a.k;
}

__global__ void __launch_bounds__(kGaThreads, 1) gather_attend_kernel(GatherAttendArgs p) {
  extern __shared__ __align__(16) unsigned char ga_smem[];
  const GatherArgs& g = p.g;
  const DecodeArgs& a = p.d;
  const bool attn = threadIdx.x >= kGaCopy;
  const int rt = attn ? threadIdx.x - kGaCopy : threadIdx.x;  // thread index within its role
  const int warp = rt >> 5, lane = threadIdx.x & 31;
  const WarpStates ws(ga_smem + kGaStages * kGaStageBytes);
  int* flag = reinterpret_cast<int*>(ga_smem + kGaStages * kGaStageBytes + kGaWsBytes);
  grid_dep_wait();  // the plan (list, count, counters) is complete and visible
  // one read of the list length and of the staged block for the whole CTA
  // (the last unit merged of the step clears the count)
  int* s_entry = flag + 4;  // entry claimed for stage 0, 1
  if (threadIdx.x == 0) {
    flag[1] = *g.count;
    // the most recently closed block may not have reached the host store yet:
    // it is read from its staging copy in HBM
    flag[2] = g.stage_k ? g.ds->staged_block : -1;
  }
  __syncthreads();
  const int count = flag[1];
  const int staged = flag[2];
  const auto attn_sync = [] { bar_sync(kBarAttn, kGaRole); };

  // Entries are claimed one at a time from a device-wide counter, so CTAs
  // that PCIe serves faster take more of them and all finish together.  The
  // copy role claims and hands the entry to the attention role with the
  // stage; a claim past the end is handed over as the signal to stop.
  if (!attn) {
    int i = 0;
    for (;; ++i) {
      const int st = i & 1;
      unsigned char* stage = ga_smem + st * kGaStageBytes;
      if (i >= kGaStages) bar_sync(kBarEmpty + st, kGaThreads);
      if (rt == 0) s_entry[st] = atomicAdd(&g.ds->gather_next, 1);
      bar_sync(kBarCopy, kGaCopy);
      const int e = s_entry[st];
      if (e >= count) {
        bar_arrive(kBarFull + st, kGaThreads);
        break;
      }
      const int4 it = g.glist[e];
      if (entry_valid(g, a, it)) {
        const bool from_stage = it.y == staged;
        const size_t src = from_stage ? (size_t)it.x * (kBlockBytes / 16)
                                      : ((size_t)it.x * g.max_blocks + it.y) * (kBlockBytes / 16);
        const size_t dst = ((size_t)it.x * g.C + it.z) * (kBlockBytes / 16);
        const uint4* sk = reinterpret_cast<const uint4*>(from_stage ? g.stage_k : g.hk) + src;
        const uint4* sv = reinterpret_cast<const uint4*>(from_stage ? g.stage_v : g.hv) + src;
        uint4* dk = reinterpret_cast<uint4*>(g.ck) + dst;
        uint4* dv = reinterpret_cast<uint4*>(g.cv) + dst;
        uint4 rk[kGaPer], rv[kGaPer];
#pragma unroll
        for (int j = 0; j < kGaPer; ++j) {
          rk[j] = ld_host(sk + rt + j * kGaCopy);
          rv[j] = ld_host(sv + rt + j * kGaCopy);
        }
#pragma unroll
        for (int j = 0; j < kGaPer; ++j) {
          const int x = rt + j * kGaCopy;  // 16-byte word x: token x / 16, chunk x % 16
          dk[x] = rk[j];
          dv[x] = rv[j];
          const uint32_t off = tile_offset(x >> 4, x & 15);
          *reinterpret_cast<uint4*>(stage + off) = rk[j];
          *reinterpret_cast<uint4*>(stage + kBlockBytes + off) = rv[j];
        }
      } else if (rt == 0) {
        atomicOr(&g.ds->error_bits, ERR_RANGE);
      }
      bar_arrive(kBarFull + st, kGaThreads);
    }
    // i entries were real; take the EMPTY arrival of the last one, the only
    // one not consumed inside the loop
    if (i >= 1) bar_sync(kBarEmpty + ((i - 1) & 1), kGaThreads);
  } else {
    for (int i = 0;; ++i) {
      const int st = i & 1;
      unsigned char* stage = ga_smem + st * kGaStageBytes;
      bar_sync(kBarFull + st, kGaThreads);
      const int e = s_entry[st];
      if (e >= count) break;
      const int4 it = g.glist[e];
      const bool valid = entry_valid(g, a, it);
      AttnAcc acc;
      acc_init(acc);
      if (valid) {
        uint32_t qf[8][2];
        load_query(a, it.x, lane, qf);
        const uint32_t kb = smem_u32(stage);
        attend_block(kb, kb + kBlockBytes, warp, lane, kP, qf, acc);
      }
      bar_arrive(kBarEmpty + st, kGaThreads);  // the stage (and its entry slot) is read out
      if (valid) {
        const int u = it.x;
        const size_t part = (size_t)u * a.nparts + a.miss_base + it.w;
        publish_warp_state(acc, ws, warp, lane, attn_sync);
        store_partial(ws, a.G, a.part_o + part * a.G * kD, a.part_ml + part * a.G, rt, kGaRole);
        contribute_partial(a, u, hits_segments(a, u), fetched_blocks(a, u), rt, kGaRole, flag, attn_sync);
      }
    }
  }
}

cudaError_t configure_gather_attend() {
  return cudaFuncSetAttribute(gather_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGaSmemBytes);
}

// Launched with the device's highest CTA priority so that its few CTAs are
// dispatched ahead of the hits pass running beside it.
cudaError_t launch_gather_attend(const GatherAttendArgs& a, int grid, cudaStream_t st, bool pdl) {
  int least = 0, greatest = 0;
  cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
  if (e != cudaSuccess) return e;
  return launch_ex(gather_attend_kernel, dim3(grid), dim3(kGaThreads), kGaSmemBytes, st, pdl, greatest, a);
}

}  // namespace nosa
