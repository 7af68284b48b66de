// attend.cu -- the hits pass: block-sparse GQA attention over the selected
// blocks that are on the GPU when the step starts.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), App. A:
// attention is computed with the GPU-resident KV blocks.  Per 64-token block
// (the math is in attend_dev.cuh), K and V (16 KiB each) are staged in shared
// memory by 2-D TMA loads with the 128-byte swizzle; three blocks are in
// flight, tracked by mbarriers.
//
// attend_hits_kernel is persistent (two CTAs per SM), stream-K style: every
// CTA walks one contiguous, equal-length range of the flattened (unit, block)
// sequence while thread 0 keeps TMA loads three blocks ahead across unit
// boundaries.  Each (unit, CTA) segment writes a partial.  With KV resident
// that is all of S(t); with KV in host memory it is S(t)'s cache hits plus the
// open tail, and the blocks fetched this step are attended by the gather
// kernel as they land (gather_attend.cu).  Whichever contributor completes a
// unit's partials merges them into the output -- no kernel waits for another.
#include "attend_dev.cuh"

namespace nosa {

constexpr int kAttnThreads = 128;
constexpr int kStageBytes = 2 * kBlockBytes;
// Shared memory of a CTA with S stages: the stages, S mbarriers, a flag word
// and slack for 1024-byte alignment.
constexpr int smem_bytes_for(int S) { return S * kStageBytes + S * 8 + 16 + 1024; }
// The producer-warp pass: S FULL and S EMPTY mbarriers.
constexpr int smem_ws_bytes_for(int S) { return S * kStageBytes + 2 * S * 8 + 16 + 1024; }
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Issue the TMA loads of one block (K and V: four 64 x 64 boxes, 32 KiB).
__device__ __forceinline__ void issue_block(const DecodeMaps& m, const DecodeArgs& a, unsigned char* sm,
                                            uint64_t* bars, int st, int u, int pos, bool tail) {
  const CUtensorMap* mk = &m.k;
  const CUtensorMap* mv = &m.v;
  int row;
  if (tail) {
    mk = &m.tk;
    mv = &m.tv;
    row = u * kP;
  } else if (a.resident) {
    int blk = a.sel[(size_t)u * a.k + pos];
    if (blk < 0 || blk >= a.max_blocks) {
      atomicOr(&a.ds->error_bits, ERR_RANGE);
      blk = 0;
    }
    row = (u * a.max_blocks + blk) * kP;
  } else {
    int slot = a.items[(size_t)u * a.k + pos];
    if (slot < 0 || slot >= a.C) {
      atomicOr(&a.ds->error_bits, ERR_RANGE);
      slot = 0;
    }
    row = (u * a.C + slot) * kP;
  }
  unsigned char* kt = sm + st * kStageBytes;
  unsigned char* vt = kt + kBlockBytes;
  mbar_arrive_expect_tx(&bars[st], 2 * kBlockBytes);
  if (a.kv_evict_first) {
    const uint64_t pol = l2_evict_first_policy();
    tma_load_2d_hint(kt, mk, &bars[st], 0, row, pol);
    tma_load_2d_hint(kt + kHalfBytes, mk, &bars[st], 64, row, pol);
    tma_load_2d_hint(vt, mv, &bars[st], 0, row, pol);
    tma_load_2d_hint(vt + kHalfBytes, mv, &bars[st], 64, row, pol);
  } else {
    tma_load_2d(kt, mk, &bars[st], 0, row);
    tma_load_2d(kt + kHalfBytes, mk, &bars[st], 64, row);
    tma_load_2d(vt, mv, &bars[st], 0, row);
    tma_load_2d(vt + kHalfBytes, mv, &bars[st], 64, row);
  }
}

__device__ __forceinline__ bool position_valid(const DecodeArgs& a, int j, int n_hit_u, int tail_len) {
  if (j < a.k) return a.resident ? true : j < n_hit_u;
  return j == a.k && tail_len > 0;  // the open tail; positions past it are the unit's gap
}

template <int kStages>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attend_hits_kernel(const __grid_constant__ DecodeMaps maps, DecodeArgs a) {
  extern __shared__ unsigned char attn_smem_raw[];
  unsigned char* sm = aligned_smem(attn_smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kStages * kStageBytes);
  int* s_flag = reinterpret_cast<int*>(sm + kStages * kStageBytes + kStages * 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tail_len = a.tail_split ? a.ds->tail_len_step : 0;
  Walk wk;
  wk.vpu = a.vpu;
  wk.V = (long long)a.U * wk.vpu;
  wk.grid = gridDim.x;
  const long long p0 = wk.start(blockIdx.x), p1 = wk.start(blockIdx.x + 1);

  // producer cursor (thread 0 only): next position to issue
  long long pp = p0;
  int pu = -1, pn_hit = 0, issued = 0;
  auto issue_next = [&](int st) {
    for (; pp < p1; ++pp) {
      const int u = (int)(pp / wk.vpu), j = (int)(pp % wk.vpu);
      if (u != pu) {
        pu = u;
        pn_hit = a.resident ? a.k : a.n_hit[u];
      }
      if (position_valid(a, j, pn_hit, tail_len)) {
        issue_block(maps, a, sm, bars, st, u, j < a.k ? j : 0, j >= a.k);
        ++issued;
        ++pp;
        return;
      }
    }
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    for (int i = 0; i < kStages; ++i) issue_next(i);
  }
  __syncthreads();

  int gb = 0;  // blocks consumed
  long long p = p0;
  while (p < p1) {
    // one segment: the positions of one unit inside this CTA's range
    const int u = (int)(p / wk.vpu);
    const long long seg_end = min(p1, (long long)(u + 1) * wk.vpu);
    const int n_hit_u = a.resident ? a.k : a.n_hit[u];
    const int first_cta = wk.cta_of((long long)u * wk.vpu);
    const int n_segs = wk.cta_of((long long)(u + 1) * wk.vpu - 1) - first_cta + 1;
    const size_t part = (size_t)u * a.nparts + a.part_base + (blockIdx.x - first_cta);
    float* po = a.part_o + part * a.G * kD;
    float2* pml = a.part_ml + part * a.G;

    uint32_t qf[8][2];
    load_query(a, u, lane, qf);
    AttnAcc acc;
    acc_init(acc);
    int consumed_here = 0;
    for (; p < seg_end; ++p) {
      const int j = (int)(p % wk.vpu);
      if (!position_valid(a, j, n_hit_u, tail_len)) continue;
      const int st = gb % kStages;
      const bool ok = mbar_wait_bounded(&bars[st], (uint32_t)((gb / kStages) & 1), kWaitLimitNs);
      if (__syncthreads_or(!ok)) {
        // record, give the loads already issued a bounded chance to land, stop
        if (threadIdx.x == 0) {
          atomicOr(&a.ds->error_bits, ERR_TIMEOUT);
          for (int g2 = gb; g2 < issued; ++g2)
            (void)mbar_wait_bounded(&bars[g2 % kStages], (uint32_t)((g2 / kStages) & 1), kWaitLimitNs);
        }
        __syncthreads();
        return;
      }
      const uint32_t kb = smem_u32(sm + st * kStageBytes);
      attend_block(kb, kb + kBlockBytes, warp, lane, j < a.k ? kP : tail_len, qf, acc);
      ++gb;
      ++consumed_here;
      __syncthreads();  // every warp is done with stage st
      // is this the segment's last valid position?
      bool last = true;
      for (long long q = p + 1; q < seg_end; ++q)
        if (position_valid(a, (int)(q % wk.vpu), n_hit_u, tail_len)) {
          last = false;
          break;
        }
      if (last) {
        // the segment's partial, merged through the stage just consumed
        const WarpStates ws(sm + st * kStageBytes);
        publish_warp_state(acc, ws, warp, lane, [] { __syncthreads(); });
        store_partial(ws, a.G, po, pml, threadIdx.x, kAttnThreads);
        __syncthreads();
      }
      if (threadIdx.x == 0) {
        fence_proxy_async_smem();
        issue_next(st);
      }
    }
    if (consumed_here == 0 && threadIdx.x < a.G) pml[threadIdx.x] = make_float2(-INFINITY, 0.f);

    // whoever completes the unit's partials (this CTA, another segment's, or
    // the gather of its last fetched block) merges them
    contribute_partial(a, u, n_segs, fetched_blocks(a, u), threadIdx.x, kAttnThreads, s_flag,
                       [] { __syncthreads(); });
  }
}

// The same pass with a producer warp of its own.  Warp 4 (one thread) walks
// the CTA's positions and keeps kStages blocks of TMA loads in flight, each
// stage guarded by a FULL mbarrier (the loads' bytes) and an EMPTY one (the
// four consumer warps); warps 0-3 attend the blocks in the same order.  A
// segment's end (its partial, the unit count, the next unit's queries) no
// longer holds up the loads: only the stage that the partial is staged
// through stays busy until it is written.  Positions are tracked as
// (unit, index) pairs instead of being divided out of a flat index, and a
// segment's last valid position is known in closed form.  Same walk, same
// partials, same arithmetic: the outputs are bit-identical to the pass above.
constexpr int kBarCons = 1;  // named barrier: the consumer warps alone

template <int kStages>
__global__ void __launch_bounds__(kAttnThreads + 32, 2)
    attend_hits_ws_kernel(const __grid_constant__ DecodeMaps maps, DecodeArgs a) {
  extern __shared__ unsigned char attn_smem_raw[];
  unsigned char* sm = aligned_smem(attn_smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  int* s_flag = reinterpret_cast<int*>(empty + kStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tail_len = a.tail_split ? a.ds->tail_len_step : 0;
  Walk wk;
  wk.vpu = a.vpu;
  wk.V = (long long)a.U * wk.vpu;
  wk.grid = gridDim.x;
  const long long p0 = wk.start(blockIdx.x), p1 = wk.start(blockIdx.x + 1);
  const int vpu = a.vpu;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);  // one arrival per consumer warp
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (p0 >= p1) return;
  const int u0 = (int)(p0 / vpu), j0 = (int)(p0 % vpu);
  const int npos = (int)(p1 - p0);

  if (warp == 4) {
    // ---- producer
    if (lane != 0) return;
    int u = u0, j = j0, issued = 0;
    int n_hit_u = a.resident ? a.k : a.n_hit[u];
    bool timed_out = false;
    for (int q = 0; q < npos; ++q) {
      if (position_valid(a, j, n_hit_u, tail_len)) {
        const int st = issued % kStages;
        if (issued >= kStages &&
            !mbar_wait_bounded(&empty[st], (uint32_t)((issued / kStages - 1) & 1), kWaitLimitNs)) {
          timed_out = true;
          break;
        }
        // the consumers' reads of this stage come before the copies into it
        fence_proxy_async_smem();
        issue_block(maps, a, sm, full, st, u, j < a.k ? j : 0, j >= a.k);
        ++issued;
      }
      if (++j == vpu) {
        j = 0;
        ++u;
        if (q + 1 < npos) n_hit_u = a.resident ? a.k : a.n_hit[u];
      }
    }
    if (timed_out) atomicOr(&a.ds->error_bits, ERR_TIMEOUT);
    // every stage's last loads land before this thread leaves
    for (int g2 = issued - 1; g2 >= 0 && g2 >= issued - kStages; --g2)
      (void)mbar_wait_bounded(&full[g2 % kStages], (uint32_t)((g2 / kStages) & 1), kWaitLimitNs);
    return;
  }

  // ---- consumers
  const auto cons_sync = [] { bar_sync(kBarCons, kAttnThreads); };
  int gb = 0;  // blocks consumed
  int u = u0, j = j0, q = 0;
  // the next segment's queries are loaded while this one streams its blocks
  uint32_t qf[8][2], qn[8][2];
  load_query(a, u, lane, qn);
  while (q < npos) {
    // one segment: the positions of unit u inside this CTA's range
    const int seg_len = min(npos - q, vpu - j);
    const int n_hit_u = a.resident ? a.k : a.n_hit[u];
    const int first_cta = wk.cta_of((long long)u * vpu);
    const int n_segs = wk.cta_of((long long)(u + 1) * vpu - 1) - first_cta + 1;
    const size_t part = (size_t)u * a.nparts + a.part_base + (blockIdx.x - first_cta);
    float* po = a.part_o + part * a.G * kD;
    float2* pml = a.part_ml + part * a.G;
    // the segment's last valid position (-1: none): the open tail if the
    // segment reaches it, else its last block in [j, j + seg_len)
    const int seg_end = j + seg_len - 1;
    int seg_last;
    if (tail_len > 0 && seg_end >= a.k && j <= a.k) {
      seg_last = a.k;
    } else {
      seg_last = min(seg_end, (a.resident ? a.k : n_hit_u) - 1);
      if (seg_last < j) seg_last = -1;
    }

#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qf[ks][0] = qn[ks][0];
      qf[ks][1] = qn[ks][1];
    }
    if (q + seg_len < npos) load_query(a, u + 1, lane, qn);
    AttnAcc acc;
    acc_init(acc);
    int consumed_here = 0;
    for (int jj = j; jj < j + seg_len; ++jj) {
      if (!position_valid(a, jj, n_hit_u, tail_len)) continue;
      const int st = gb % kStages;
      const bool ok = mbar_wait_bounded(&full[st], (uint32_t)((gb / kStages) & 1), kWaitLimitNs);
      if (bar_red_or(kBarCons, kAttnThreads, !ok)) {
        if (threadIdx.x == 0) atomicOr(&a.ds->error_bits, ERR_TIMEOUT);
        return;
      }
      const uint32_t kb = smem_u32(sm + st * kStageBytes);
      attend_block(kb, kb + kBlockBytes, warp, lane, jj < a.k ? kP : tail_len, qf, acc);
      ++gb;
      ++consumed_here;
      if (jj == seg_last) {
        // the segment's partial, merged through the stage just consumed
        cons_sync();  // every consumer warp is done reading the stage
        const WarpStates ws(sm + st * kStageBytes);
        publish_warp_state(acc, ws, warp, lane, cons_sync);
        store_partial(ws, a.G, po, pml, threadIdx.x, kAttnThreads);
        cons_sync();
      } else {
        __syncwarp();
      }
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (consumed_here == 0 && threadIdx.x < a.G) pml[threadIdx.x] = make_float2(-INFINITY, 0.f);

    // whoever completes the unit's partials (this CTA, another segment's, or
    // the gather of its last fetched block) merges them
    contribute_partial(a, u, n_segs, fetched_blocks(a, u), threadIdx.x, kAttnThreads, s_flag, cons_sync);
    q += seg_len;
    j = 0;
    ++u;
  }
}

// Partial slots a unit needs in the hits pass for a grid of `grid` CTAs.
__host__ __device__ inline int hits_segments_per_unit(int U, int vpu, int grid) {
  // a unit spans at most ceil(vpu * grid / V) + 1 CTA ranges, V = U * vpu
  const long long V = (long long)U * vpu;
  return (int)(((long long)vpu * grid + V - 1) / V) + 1;
}

// Called once per context creation (on its device), outside any stream capture.
cudaError_t configure_decode() {
  cudaError_t e = cudaFuncSetAttribute(attend_hits_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem_bytes_for(3));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attend_hits_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes_for(2));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attend_hits_ws_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_ws_bytes_for(3));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attend_hits_ws_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_ws_bytes_for(2));
  if (e != cudaSuccess) return e;

  return configure_gather_attend();
}

// stages: TMA stages per CTA (2 or 3); the grid's CTAs per SM follow from it.
cudaError_t launch_attend_hits(const DecodeArgs& a, const DecodeMaps& m, int grid, cudaStream_t st, int stages,
                               bool producer_warp) {
  if (producer_warp) {
    if (stages == 2) {
      attend_hits_ws_kernel<2><<<grid, kAttnThreads + 32, smem_ws_bytes_for(2), st>>>(m, a);
    } else {
      attend_hits_ws_kernel<3><<<grid, kAttnThreads + 32, smem_ws_bytes_for(3), st>>>(m, a);
    }
    return cudaGetLastError();
  }
  if (stages == 2) {
    attend_hits_kernel<2><<<grid, kAttnThreads, smem_bytes_for(2), st>>>(m, a);
  } else {
    attend_hits_kernel<3><<<grid, kAttnThreads, smem_bytes_for(3), st>>>(m, a);
  }
  return cudaGetLastError();
}

int attend_hits_grid(int U, int vpu, int want) {
  const long long V = (long long)U * vpu;
  if (want > V) want = (int)V;
  return want < 1 ? 1 : want;
}

int attend_hits_parts(int U, int vpu, int grid) {
  return hits_segments_per_unit(U, vpu, attend_hits_grid(U, vpu, grid));
}

}  // namespace nosa
