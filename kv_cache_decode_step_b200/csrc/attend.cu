// attend.cu -- block-sparse GQA attention over the selected blocks.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), App. A:
// after the misses arrive, attention is computed with the GPU-resident KV
// blocks.  Each query head attends to the 64 tokens of every selected block of
// its KV head (plus the open tail block), softmax scaled by 1/sqrt(d).
//
// Per 64-token block (shared by both kernels below):
//  * K and V (16 KiB each) are staged in shared memory by 2-D TMA loads with
//    the 128-byte swizzle; three blocks are in flight, tracked by mbarriers.
//  * Four warps each own 16 tokens.  Scores S^T[token][head] come from
//    mma.m16n8k16 with the block as A (tokens x dims) and the query group as B
//    (dims x 8 heads; heads >= G are zero), so the 4-head group wastes half of
//    N rather than 3/4 of M.  P^T is moved into the B layout with movmatrix and
//    O^T[dim][head] += V^T P^T uses ldmatrix.trans on the V tile.
//  * Online softmax per warp in the exp2 domain; warps, then splits, are
//    merged with log-sum-exp weights.
//
// Kernels:
//  * attend_hits_kernel: persistent (two CTAs per SM), stream-K style: every
//    CTA walks one contiguous, equal-length range of the flattened (unit,
//    block) sequence while thread 0 keeps TMA loads three blocks ahead across
//    unit boundaries.  Each (unit, CTA) segment writes a partial; with KV
//    resident, the last CTA to finish a segment of a unit merges its partials
//    into the output (no waiting: the others simply move on).
//  * attend_misses_kernel: one CTA per unit over the blocks fetched this step,
//    launched after the gather; it merges every partial of the unit.
#include "nosa_internal.cuh"

namespace nosa {

constexpr int kStages = 3;
constexpr int kAttnThreads = 128;
constexpr int kHalfBytes = kP * 64 * 2;  // one 64-row x 64-dim box = 8 KiB
constexpr int kStageBytes = 2 * kBlockBytes;
constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kFlagOffset = kBarOffset + kStages * 8;
constexpr int kSmemBytes = kFlagOffset + 16 + 1024;  // + slack for 1024-byte alignment
// The misses pass holds one block at a time (a unit misses 0-3 blocks in the
// steady state), so six of its CTAs fit per SM and the whole batch runs in one
// wave; its warp states reuse the single stage.
constexpr int kMissStages = 1;
constexpr int kMissBarOffset = kMissStages * kStageBytes;
constexpr int kMissSmemBytes = kMissBarOffset + 16 + 1024;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kScoreScale = 0.088388347648318440f * 1.4426950408889634f;  // log2(e) / sqrt(128)

struct AttnAcc {
  float o[8][4];  // O^T fragments: dims 16 mt + lane/4 (+8), heads 2 (lane%4) (+1)
  float m0, m1, l0, l1;
};

__device__ __forceinline__ void acc_init(AttnAcc& s) {
#pragma unroll
  for (int i = 0; i < 8; ++i) s.o[i][0] = s.o[i][1] = s.o[i][2] = s.o[i][3] = 0.f;
  s.m0 = s.m1 = -INFINITY;
  s.l0 = s.l1 = 0.f;
}

__device__ __forceinline__ unsigned char* aligned_smem(unsigned char* raw) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The query group of unit u as the mma B operand: lane holds head lane/4,
// dims 16 ks + 2 (lane%4) + {0,1} and + 8.
__device__ __forceinline__ void load_query(const DecodeArgs& a, int u, int lane, uint32_t (&qf)[8][2]) {
  const int b = u / a.Hkv, g = u % a.Hkv;
  const int hb = lane >> 2;
  const uint32_t* qrow =
      reinterpret_cast<const uint32_t*>(a.q + ((size_t)b * a.Hq + (size_t)g * a.G + (hb < a.G ? hb : 0)) * kD);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    qf[ks][0] = hb < a.G ? qrow[ks * 8 + (lane & 3)] : 0u;
    qf[ks][1] = hb < a.G ? qrow[ks * 8 + 4 + (lane & 3)] : 0u;
  }
}

// One 64-token block from shared memory (kb, vb: K and V tile addresses);
// tokens at or beyond len are masked out.
__device__ __forceinline__ void attend_block(uint32_t kb, uint32_t vb, int warp, int lane, int len,
                                             const uint32_t (&qf)[8][2], AttnAcc& s) {
  const int tok_a = warp * 16 + (lane & 15);                       // ldmatrix row, K
  const int tok_v = warp * 16 + (lane & 7) + ((lane >> 4) << 3);  // ldmatrix row, V (trans)
  const int t0 = warp * 16 + (lane >> 2), t1 = t0 + 8;             // accumulator rows
  float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int chunk = 2 * ks + (lane >> 4);
    const uint32_t addr = kb + (chunk >> 3) * kHalfBytes + tok_a * 128 + (((chunk & 7) ^ (tok_a & 7)) << 4);
    uint32_t a0, a1, a2, a3;
    ldsm_x4(addr, a0, a1, a2, a3);
    mma_bf16_16816(c, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
  }
  const float s0 = t0 < len ? c[0] * kScoreScale : -INFINITY;
  const float s1 = t0 < len ? c[1] * kScoreScale : -INFINITY;
  const float s2 = t1 < len ? c[2] * kScoreScale : -INFINITY;
  const float s3 = t1 < len ? c[3] * kScoreScale : -INFINITY;
  float bm0 = fmaxf(s0, s2), bm1 = fmaxf(s1, s3);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
    bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
  }
  const float mn0 = fmaxf(s.m0, bm0), mn1 = fmaxf(s.m1, bm1);
  const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
  const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
  const float al0 = exp2f(s.m0 - mu0), al1 = exp2f(s.m1 - mu1);
  const float p0 = exp2f(s0 - mu0), p1 = exp2f(s1 - mu1);
  const float p2 = exp2f(s2 - mu0), p3 = exp2f(s3 - mu1);
  s.l0 = s.l0 * al0 + p0 + p2;
  s.l1 = s.l1 * al1 + p1 + p3;
  s.m0 = mn0;
  s.m1 = mn1;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    s.o[mt][0] *= al0; s.o[mt][1] *= al1; s.o[mt][2] *= al0; s.o[mt][3] *= al1;
  }
  const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
  const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int chunk = 2 * mt + ((lane >> 3) & 1);
    const uint32_t addr = vb + (chunk >> 3) * kHalfBytes + tok_v * 128 + (((chunk & 7) ^ (tok_v & 7)) << 4);
    uint32_t a0, a1, a2, a3;
    ldsm_x4_trans(addr, a0, a1, a2, a3);
    mma_bf16_16816(s.o[mt], a0, a1, a2, a3, pb0, pb1);
  }
}

// Shared-memory view of the four warps' states: sO [4][8][128], sM, sL [4][8].
struct WarpStates {
  float* o;
  float* m;
  float* l;
  __device__ explicit WarpStates(unsigned char* buf)
      : o(reinterpret_cast<float*>(buf)), m(o + 4 * kMaxG * kD), l(m + 4 * kMaxG) {}
};

// Every thread: publish this warp's state into ws (ends with __syncthreads).
__device__ __forceinline__ void publish_warp_state(AttnAcc& s, const WarpStates& ws, int warp, int lane) {
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    s.l0 += __shfl_xor_sync(0xffffffffu, s.l0, off);
    s.l1 += __shfl_xor_sync(0xffffffffu, s.l1, off);
  }
  const int h0 = (lane & 3) * 2, h1 = h0 + 1;
  if (lane < 4) {
    ws.m[warp * kMaxG + h0] = s.m0; ws.m[warp * kMaxG + h1] = s.m1;
    ws.l[warp * kMaxG + h0] = s.l0; ws.l[warp * kMaxG + h1] = s.l1;
  }
  float* w = ws.o + warp * kMaxG * kD;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d0 = mt * 16 + (lane >> 2);
    w[h0 * kD + d0] = s.o[mt][0];
    w[h1 * kD + d0] = s.o[mt][1];
    w[h0 * kD + d0 + 8] = s.o[mt][2];
    w[h1 * kD + d0 + 8] = s.o[mt][3];
  }
  __syncthreads();
}

// Merge the four warps' states into one partial (unnormalised O, max, sum).
__device__ __forceinline__ void store_partial(const WarpStates& ws, int G, float* po, float2* pml) {
  for (int idx = threadIdx.x; idx < G * kD; idx += kAttnThreads) {
    const int h = idx / kD, dd = idx % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, ws.m[w * kMaxG + h]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float f = exp2f(ws.m[w * kMaxG + h] - Mu);
      acc += f * ws.o[(w * kMaxG + h) * kD + dd];
      L += f * ws.l[w * kMaxG + h];
    }
    po[h * kD + dd] = acc;
    if (dd == 0) pml[h] = make_float2(M, L);
  }
}

// Running log-sum-exp merge of (max m, sum l, accumulator o) triples.
struct LseMerge {
  float M = -INFINITY, num = 0.f, den = 0.f;
  __device__ __forceinline__ void add(float m, float l, float o) {
    if (!(l > 0.f)) return;
    if (m > M) {
      const float s = exp2f(M - m);  // M = -inf gives 0
      num *= s;
      den *= s;
      M = m;
    }
    const float f = exp2f(m - M);
    num += f * o;
    den += f * l;
  }
};

// out[b, g*G + h, :] = merge of the unit's partials [0, nparts) (read around
// L1: other CTAs wrote them) and, optionally, this CTA's warp states.  Thread
// d owns dim d; heads go two at a time, with the loads of four parts of both
// issued together.
__device__ void merge_unit(const DecodeArgs& a, int u, int nparts, const WarpStates* ws) {
  const int b = u / a.Hkv, g = u % a.Hkv;
  const float* po = a.part_o + (size_t)u * a.nparts * a.G * kD;
  const float2* pml = a.part_ml + (size_t)u * a.nparts * a.G;
  for (int dd = threadIdx.x; dd < kD; dd += blockDim.x) {
    for (int h0 = 0; h0 < a.G; h0 += 2) {
      LseMerge mg[2];
      for (int p0 = 0; p0 < nparts; p0 += 4) {
        float2 ml[4][2];
        float ov[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = h0 + e;
            const bool on = p0 + i < nparts && h < a.G;
            ml[i][e] = on ? __ldcg(&pml[(p0 + i) * a.G + h]) : make_float2(-INFINITY, 0.f);
            ov[i][e] = on ? __ldcg(&po[((size_t)(p0 + i) * a.G + h) * kD + dd]) : 0.f;
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mg[0].add(ml[i][0].x, ml[i][0].y, ov[i][0]);
          mg[1].add(ml[i][1].x, ml[i][1].y, ov[i][1]);
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = h0 + e;
        if (h >= a.G) break;
        if (ws) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
            mg[e].add(ws->m[w * kMaxG + h], ws->l[w * kMaxG + h], ws->o[(w * kMaxG + h) * kD + dd]);
        }
        const float r = mg[e].den > 0.f ? mg[e].num / mg[e].den : 0.f;
        a.out[((size_t)b * a.Hq + (size_t)g * a.G + h) * kD + dd] = (uint16_t)(pack_bf16x2(r, 0.f) & 0xFFFFu);
      }
    }
  }
}

// Every CTA calls this once at its very end: the last one to arrive ends the
// step (all other CTAs of the kernel are done with the state by then).
__device__ __forceinline__ void finish_step(const DecodeArgs& a) {
  if (!a.done_ctr) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0 && atomicAdd(a.done_ctr, 1) == (int)(gridDim.x * gridDim.y) - 1) {
    __threadfence();
    advance_step(a.ds, a.st);
    *a.done_ctr = 0;
  }
}

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
  tma_load_2d(kt, mk, &bars[st], 0, row);
  tma_load_2d(kt + kHalfBytes, mk, &bars[st], 64, row);
  tma_load_2d(vt, mv, &bars[st], 0, row);
  tma_load_2d(vt + kHalfBytes, mv, &bars[st], 64, row);
}

// The hits pass walks a virtual sequence of positions: unit u owns positions
// [u * vpu, (u + 1) * vpu), vpu = k + tail_split; position j < k of unit u is
// its j-th selected block (valid when j < k with KV resident, j < n_hit[u]
// otherwise) and position k is its open tail (valid when it holds tokens).
// CTA c takes the contiguous range [start(c), start(c + 1)), start(c) =
// floor(c * V / grid), so every CTA streams the same number of positions and
// touches one to a few units; each (unit, CTA) segment writes one partial.
struct Walk {
  long long V;
  int vpu, grid;
  __device__ long long start(int c) const { return (long long)c * V / grid; }
  // the CTA whose range holds position p
  __device__ int cta_of(long long p) const { return (int)(((p + 1) * grid - 1) / V); }
};

__device__ __forceinline__ bool position_valid(const DecodeArgs& a, int j, int n_hit_u, int tail_len) {
  if (j < a.k) return a.resident ? true : j < n_hit_u;
  return tail_len > 0;
}

__global__ void __launch_bounds__(kAttnThreads, 2)
    attend_hits_kernel(const __grid_constant__ DecodeMaps maps, DecodeArgs a) {
  extern __shared__ unsigned char attn_smem_raw[];
  unsigned char* sm = aligned_smem(attn_smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kBarOffset);
  int* s_flag = reinterpret_cast<int*>(sm + kFlagOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tail_len = a.tail_split ? a.ds->tail_len_step : 0;
  Walk wk;
  wk.vpu = a.k + a.tail_split;
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
        publish_warp_state(acc, ws, warp, lane);
        store_partial(ws, a.G, po, pml);
        __syncthreads();
      }
      if (threadIdx.x == 0) {
        fence_proxy_async_smem();
        issue_next(st);
      }
    }
    if (consumed_here == 0 && threadIdx.x < a.G) pml[threadIdx.x] = make_float2(-INFINITY, 0.f);

    if (a.unit_done) {
      // the last CTA to finish a segment of the unit merges all of them
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) *s_flag = (atomicAdd(&a.unit_done[u], 1) == n_segs - 1);
      __syncthreads();
      if (*s_flag) {
        __threadfence();
        merge_unit(a, u, n_segs, nullptr);
        if (threadIdx.x == 0) a.unit_done[u] = 0;
      }
      __syncthreads();
    }
  }
  finish_step(a);
}

// Partial slots a unit needs in the hits pass for a grid of `grid` CTAs.
__host__ __device__ inline int hits_segments_per_unit(int U, int vpu, int grid) {
  // a unit spans at most ceil(vpu * grid / V) + 1 CTA ranges, V = U * vpu
  const long long V = (long long)U * vpu;
  return (int)(((long long)vpu * grid + V - 1) / V) + 1;
}

// One CTA per unit: the blocks fetched this step (one at a time), then the
// merge of every partial of the unit into the output.
__global__ void __launch_bounds__(kAttnThreads)
    attend_misses_kernel(const __grid_constant__ DecodeMaps maps, DecodeArgs a) {
  extern __shared__ unsigned char attn_smem_raw[];
  unsigned char* sm = aligned_smem(attn_smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kMissBarOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x;
  const int lo = a.n_hit[u], hi = a.n_items[u];
  const int n = hi > lo ? hi - lo : 0;
  // the hits pass wrote one partial per (unit, CTA) segment
  Walk wk;
  wk.vpu = a.k + a.tail_split;
  wk.V = (long long)a.U * wk.vpu;
  wk.grid = a.hits_grid;
  const int n_segs = wk.cta_of((long long)(u + 1) * wk.vpu - 1) - wk.cta_of((long long)u * wk.vpu) + 1;
  if (n == 0) {
    merge_unit(a, u, n_segs, nullptr);
    finish_step(a);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    issue_block(maps, a, sm, bar, 0, u, lo, false);
  }
  __syncthreads();
  uint32_t qf[8][2];
  load_query(a, u, lane, qf);
  AttnAcc acc;
  acc_init(acc);
  const uint32_t kb = smem_u32(sm);
  for (int j = 0; j < n; ++j) {
    const bool ok = mbar_wait_bounded(bar, (uint32_t)(j & 1), kWaitLimitNs);
    if (__syncthreads_or(!ok)) {
      if (threadIdx.x == 0) atomicOr(&a.ds->error_bits, ERR_TIMEOUT);
      __syncthreads();
      return;
    }
    attend_block(kb, kb + kBlockBytes, warp, lane, kP, qf, acc);
    __syncthreads();
    if (threadIdx.x == 0 && j + 1 < n) {
      fence_proxy_async_smem();
      issue_block(maps, a, sm, bar, 0, u, lo + j + 1, false);
    }
  }
  // every load has been consumed: the stage holds the warp states
  const WarpStates ws(sm);
  publish_warp_state(acc, ws, warp, lane);
  merge_unit(a, u, n_segs, &ws);
  finish_step(a);
}

int attend_smem_bytes() { return kSmemBytes; }

// Called once per context creation (on its device), outside any stream capture.
cudaError_t configure_decode() {
  cudaError_t e = cudaFuncSetAttribute(attend_hits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(attend_misses_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMissSmemBytes);
}

cudaError_t launch_attend_hits(const DecodeArgs& a, const DecodeMaps& m, int grid, cudaStream_t st) {
  attend_hits_kernel<<<grid, kAttnThreads, kSmemBytes, st>>>(m, a);
  return cudaGetLastError();
}

int attend_hits_grid(int U, int k, int tail_split, int want) {
  const long long V = (long long)U * (k + tail_split);
  if (want > V) want = (int)V;
  return want < 1 ? 1 : want;
}

int attend_hits_parts(int U, int k, int tail_split, int grid) {
  return hits_segments_per_unit(U, k + tail_split, attend_hits_grid(U, k, tail_split, grid));
}

cudaError_t launch_attend_misses(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t st) {
  attend_misses_kernel<<<a.U, kAttnThreads, kMissSmemBytes, st>>>(m, a);
  return cudaGetLastError();
}

}  // namespace nosa
