// prepare.cu -- the first three stages of a decode step fused into one
// kernel: block scores, selection and the cache plan of each unit.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary): §3.1
// (scores from pooled keys; selection of query-aware and query-agnostic blocks under a
// minimum overlap), §4 (set difference against the GPU-resident blocks and a
// replacement mapping).  The arithmetic is that of score_kernel,
// select_reg_kernel and the planning kernels: the same device functions run
// here, only the launch boundaries between them are gone.  One CTA owns one
// unit: its 4, 8 or 16 warps score every closed block (scores kept in shared
// memory), then warp 0 selects and plans while, with KV in HBM, warp 1 warms
// L2 for the hits pass.  The gather can start as soon as this single launch
// ends instead of after three launches in a row.
#include "plan_dev.cuh"
#include "score_dev.cuh"
#include "select_dev.cuh"

namespace nosa {

constexpr int kPrepMaxThreads = 512;

// Warp-wide: L2 prefetches of the first warm_blocks positions of every
// hits-pass CTA whose range starts in unit u, with the block ids of S(t-1)
// (prev: the unit's copy in shared memory).  The hits pass walks positions
// u * vpu + j (j < k: the j-th selected block) and CTA c starts at
// floor(c * U * vpu / grid).  A hint only: nothing reads what it brings in
// unless the pass loads the same block.
__device__ __forceinline__ void warm_first_blocks(const PrepareArgs& a, int u, int lane, const int* prev) {
  if (a.sc.ds->step == 0) return;  // no S(t-1) yet
  const long long V = (long long)a.sc.U * a.hits_vpu;
  const long long p0 = (long long)u * a.hits_vpu, p1 = p0 + a.hits_vpu;
  const int c0 = (int)((p0 * a.hits_grid + V - 1) / V);  // first CTA with start >= p0
  for (int i = lane;; i += 32) {
    const int c = c0 + i / a.warm_blocks;
    if (c >= a.hits_grid) break;
    const long long s = (long long)c * V / a.hits_grid;
    if (s >= p1) break;
    const long long p = s + i % a.warm_blocks;
    if (p >= (long long)(c + 1) * V / a.hits_grid) continue;
    const int j = (int)(p - p0);
    if (j >= a.se.k) continue;
    const int blk = prev[j];
    if (blk < 0 || blk >= a.sc.max_blocks) continue;
    const size_t off = ((size_t)u * a.sc.max_blocks + blk) * kP * kD;
    bulk_prefetch_l2(a.warm_k + off, kBlockBytes);
    bulk_prefetch_l2(a.warm_v + off, kBlockBytes);
  }
}

// Shared memory: the unit's query rows [G][16] uint4 (staged when they are
// read from host memory), scores [max_blocks] fp64, selection bitmaps [2][R] words,
// plan scratch (max(32, 2C + 2k) ints), then copies of the unit's S(t-1) [k],
// Gamma_e(t-1) [k_e], the new selection [k], the register plan's slot tables
// [32] x 2 and the general plan's block -> slot table [max_blocks].  The
// copies are loaded while the scores stream in, so selection and planning
// read no global memory of their own.
template <int R>
__global__ void __launch_bounds__(kPrepMaxThreads, 1) prepare_kernel(PrepareArgs a) {
  extern __shared__ __align__(16) unsigned char prep_smem[];
  const int k = a.se.k, ke = a.se.k_e, C = a.pl.C;
  uint4* s_q = reinterpret_cast<uint4*>(prep_smem);  // the unit's query rows when they are staged
  double* ssc = reinterpret_cast<double*>(s_q + kMaxG * kRowU4);
  unsigned(*sbm)[R] = reinterpret_cast<unsigned(*)[R]>(ssc + a.sc.max_blocks);
  int* psm = reinterpret_cast<int*>(sbm + 2);
  int* s_prev = psm + a.plan_ints;
  int* s_ge = s_prev + k;
  int* s_sel = s_ge + ke;
  int* s_sb = s_sel + k;
  int* s_lu = s_sb + 32;
  int* s_bs = s_lu + 32;  // general plan: the unit's block -> slot table [max_blocks]
  const int u = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the gather that follows may be placed now: it waits for this kernel's
  // completion before it reads anything
  grid_dep_launch();
  // the gather that follows claims its entries from 0 (it is the only user
  // of this counter and runs after this kernel has completed)
  if (u == 0 && threadIdx.x == 0) a.sc.ds->gather_next = 0;
  const bool reg_plan = a.offloaded && C <= 32 && k <= 32;

  // asynchronous copies: they land while the scores stream in
  for (int i = threadIdx.x; i < k; i += blockDim.x) cp_async4(s_prev + i, a.se.prev + (size_t)u * k + i);
  for (int i = threadIdx.x; i < ke; i += blockDim.x) cp_async4(s_ge + i, a.se.ge + (size_t)u * ke + i);
  if (reg_plan) {
    for (int i = threadIdx.x; i < C; i += blockDim.x) {
      cp_async4(s_sb + i, a.pl.slot_block + (size_t)u * C + i);
      cp_async4(s_lu + i, a.pl.last_used + (size_t)u * C + i);
    }
  } else if (a.offloaded) {
    // the general plan's slot tables go where it keeps them (psm)
    for (int i = threadIdx.x; i < C; i += blockDim.x) {
      cp_async4(psm + i, a.pl.slot_block + (size_t)u * C + i);
      cp_async4(psm + C + i, a.pl.last_used + (size_t)u * C + i);
    }
    for (int i = threadIdx.x; i < a.pl.max_blocks; i += blockDim.x)
      cp_async4(s_bs + i, a.pl.block_slot + (size_t)u * a.pl.max_blocks + i);
  }

  score_unit_warps(a.sc, u, warp, blockDim.x >> 5, lane, ssc, s_q);
  cp_async_wait_all();
  __syncthreads();
  if (warp != 0) {
    if (warp == 1 && a.warm_k) warm_first_blocks(a, u, lane, s_prev);
    return;
  }

  select_unit_reg<R>(a.se, u, lane, sbm, ssc, s_prev, s_ge, s_sel);
  __syncwarp();  // the selection is read back by the plan

  if (reg_plan) {
    plan_unit_reg(a.pl, u, lane, psm, s_sel, s_sb, s_lu);
  } else if (a.offloaded) {
    plan_unit_smem(a.pl, u, lane, psm, s_sel, s_bs, true);
  } else {
    for (int i = lane; i < k; i += 32) a.pl.fetch[(size_t)u * k + i] = -1;
    if (lane == 0) a.pl.n_fetch[u] = 0;
  }
}

template <int R>
cudaError_t launch_prepare_r(PrepareArgs a, cudaStream_t st) {
  a.plan_ints = a.offloaded ? max(32, 2 * a.pl.C + 2 * a.pl.k) : 0;
  const size_t smem = kMaxG * kRowU4 * sizeof(uint4) + (size_t)a.sc.max_blocks * sizeof(double) +
                      2 * R * sizeof(unsigned) +
                      (size_t)(a.plan_ints + 2 * a.se.k + a.se.k_e + 64) * sizeof(int) +
                      (a.offloaded ? (size_t)a.pl.max_blocks * sizeof(int) : 0);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(prepare_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int threads = 32 * max(4, min(a.nwarps, kPrepMaxThreads / 32));
  prepare_kernel<R><<<a.sc.U, threads, smem, st>>>(a);
  return cudaGetLastError();
}

bool prepare_supported(int max_blocks) { return max_blocks <= kPrepareMaxBlocks; }

// Beyond kPrepareMaxBlocks the scores come from score_kernel (many CTAs per
// unit); selection and plan then still run as one launch, one CTA per unit:
// its kSelPlanWarps warps select together (the group path of select_dev.cuh,
// 8 or 4 rows of the unit's up to 1024 blocks per lane), then warp 0 plans
// from a copy of the selection in shared memory.  The unit's scores arrive in
// shared memory in one burst of 16-byte copies before the selection reads
// them; its slot tables (and, for the general plan, its block -> slot table)
// arrive by cp.async while the selection runs, so the plan reads no global
// memory of its own.  Shared memory: the scores [sc_stride] fp64, then
// (wide_ints) the selection [k], then the general plan's scratch (2C + 2k
// ints, slot tables first) and block -> slot table [max_blocks], or the
// register plan's slot tables [32] x 2.
constexpr int kSelPlanWarps = 4;

template <int R>
__global__ void __launch_bounds__(kSelPlanWarps * 32) select_plan_kernel(SelectArgs se, PlanArgs pl, int offloaded,
                                                                        int wide_ints, int sc_stride) {
  constexpr int RW = R / kSelPlanWarps;
  extern __shared__ __align__(16) double sp_smem_d[];
  __shared__ unsigned sbm[2 * R];
  __shared__ unsigned red[2 * kSelPlanWarps * 4];
  __shared__ int ssrc[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x;
  grid_dep_wait();    // the scores are complete
  grid_dep_launch();  // the gather that follows may be placed
  // the gather that follows claims its entries from 0
  if (blockIdx.x == 0 && threadIdx.x == 0) se.ds->gather_next = 0;
  const int C = pl.C;
  const bool reg_plan = offloaded && C <= 32 && pl.k <= 32;
  double* s_sc = sp_smem_d;
  int* s_sel = reinterpret_cast<int*>(sp_smem_d + sc_stride);
  {
    // the unit's closed blocks' scores, in a copy group of their own
    const int n = se.ds->n_closed;
    const double* g_sc = se.scores + (size_t)u * se.max_blocks;
    if ((reinterpret_cast<uintptr_t>(g_sc) & 15) == 0 && (se.max_blocks & 1) == 0) {
      for (int c = threadIdx.x; c < (n + 1) / 2; c += blockDim.x) cp_async16(s_sc + 2 * c, g_sc + 2 * c);
    } else {
      for (int j = threadIdx.x; j < n; j += blockDim.x) cp_async8(s_sc + j, g_sc + j);
    }
    cp_async_commit();
  }
  int* s_plan = s_sel + se.k;                 // general plan: slot tables, then its scratch
  int* s_bs = s_plan + 2 * C + 2 * pl.k;      // general plan: block -> slot
  int* s_sb = s_plan;                         // register plan: slot -> block [32]
  int* s_lu = s_plan + 32;                    //                slot -> last step [32]
  if (offloaded && warp == 0) {
    for (int i = lane; i < C; i += 32) {
      cp_async4(s_sb + i, pl.slot_block + (size_t)u * C + i);
      cp_async4((reg_plan ? s_lu : s_plan + C) + i, pl.last_used + (size_t)u * C + i);
    }
    if (!reg_plan)
      for (int i = lane; i < pl.max_blocks; i += 32) cp_async4(s_bs + i, pl.block_slot + (size_t)u * pl.max_blocks + i);
  }
  cp_async_commit();
  cp_async_wait_group<1>();  // this thread's score copies (the tables may still be on their way)
  __syncthreads();           // and everyone else's
  SelGroup<kSelPlanWarps> g{red, warp, lane, 1};
  select_unit_group<RW, kSelPlanWarps>(se, u, g, sbm, s_sc, se.prev + (size_t)u * se.k, se.ge + (size_t)u * se.k_e,
                                       s_sel);
  cp_async_wait_all();
  __syncthreads();  // the selection and the tables are read back by the plan
  if (warp != 0) return;
  if (!offloaded) {
    for (int i = lane; i < se.k; i += 32) pl.fetch[(size_t)u * se.k + i] = -1;
    if (lane == 0) pl.n_fetch[u] = 0;
  } else if (reg_plan) {
    plan_unit_reg(pl, u, lane, ssrc, s_sel, s_sb, s_lu);
  } else {
    plan_unit_smem(pl, u, lane, s_plan, s_sel, s_bs, true);
  }
}

template <int R>
cudaError_t launch_select_plan_r(const SelectArgs& se, const PlanArgs& pl, int offloaded, cudaStream_t st,
                                 bool pdl) {
  const bool reg_plan = offloaded && pl.C <= 32 && pl.k <= 32;
  const int wide_ints = se.k + (!offloaded ? 0 : reg_plan ? 64 : 2 * pl.C + 2 * pl.k + pl.max_blocks);
  const int sc_stride = (se.max_blocks + 1) & ~1;
  const size_t smem = sc_stride * sizeof(double) + (size_t)wide_ints * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(select_plan_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_ex(select_plan_kernel<R>, dim3(se.U), dim3(kSelPlanWarps * 32), smem, st, pdl, 0, se, pl, offloaded,
                   wide_ints, sc_stride);
}

bool select_plan_supported(int max_blocks) { return max_blocks <= 1024; }

cudaError_t launch_select_plan(const SelectArgs& se, const PlanArgs& pl, int offloaded, cudaStream_t st,
                               bool pdl) {
  const int rows = (se.max_blocks + 31) / 32;
  if (rows <= 16) return launch_select_plan_r<16>(se, pl, offloaded, st, pdl);
  if (rows <= 32) return launch_select_plan_r<32>(se, pl, offloaded, st, pdl);
  return cudaErrorInvalidValue;
}

cudaError_t launch_prepare(const PrepareArgs& a, cudaStream_t st) {
  const int rows = (a.sc.max_blocks + 31) / 32;
  if (rows <= 2) return launch_prepare_r<2>(a, st);
  if (rows <= 4) return launch_prepare_r<4>(a, st);
  if (rows <= 8) return launch_prepare_r<8>(a, st);
  if (rows <= 16) return launch_prepare_r<16>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nosa
