// attend_dev.cuh -- attention of one 64-token block and the merge of a unit's
// partials, shared by the hits pass and the fused gather + attention kernel.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), App. A:
// each query head attends to the 64 tokens of every selected block of its KV
// head (plus the open tail block), softmax scaled by 1/sqrt(d).  Per block,
// four warps each own 16 tokens: scores S^T[token][head] come from
// mma.m16n8k16 with the block as A (tokens x dims) and the query group as B
// (dims x 8 heads, heads >= G zero), P^T is moved into the B layout with
// movmatrix and O^T[dim][head] += V^T P^T uses ldmatrix.trans.  Online
// softmax in the exp2 domain; warps, then partials, are merged with
// log-sum-exp weights.
//
// Shared-memory tile layout (what the 2-D TMA loads with the 128-byte swizzle
// produce): K and V of a block are two 64-token x 64-dim halves of 8 KiB;
// 16-byte chunk c (0..15) of token t sits at (c / 8) * 8 KiB + t * 128 +
// ((c % 8) ^ (t % 8)) * 16.
#pragma once

#include "nosa_internal.cuh"

namespace nosa {

constexpr int kHalfBytes = kP * 64 * 2;  // one 64-row x 64-dim box = 8 KiB
constexpr float kScoreScale = 0.088388347648318440f * 1.4426950408889634f;  // log2(e) / sqrt(128)

// byte offset of 16-byte chunk c of token t in a K or V tile
__device__ __forceinline__ uint32_t tile_offset(int t, int c) {
  return (uint32_t)((c >> 3) * kHalfBytes + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

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

// Every thread of the four attention warps: publish this warp's state into ws
// (ends with sync(), a barrier over those warps).
template <class Sync>
__device__ __forceinline__ void publish_warp_state(AttnAcc& s, const WarpStates& ws, int warp, int lane, Sync sync) {
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
  sync();
}

// Merge the four warps' states into one partial (unnormalised O, max, sum).
__device__ __forceinline__ void store_partial(const WarpStates& ws, int G, float* po, float2* pml, int tid,
                                              int nthr) {
  for (int idx = tid; idx < G * kD; idx += nthr) {
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

// out[b, g*G + h, :] = merge of unit u's partials -- the hits pass's segments
// [0, n_seg) and the fetched blocks' [miss_base, miss_base + n_miss) -- read
// around L1 (other CTAs wrote them), and optionally warp states ws.  Thread
// tid (of nthr) owns dims tid, tid + nthr, ...; heads go two at a time, with
// the loads of four parts of both issued together.
__device__ inline void merge_unit(const DecodeArgs& a, int u, int n_seg, int n_miss, const WarpStates* ws, int tid,
                           int nthr) {
  const int b = u / a.Hkv, g = u % a.Hkv;
  const float* po = a.part_o + (size_t)u * a.nparts * a.G * kD;
  const float2* pml = a.part_ml + (size_t)u * a.nparts * a.G;
  const int np = n_seg + n_miss;
  for (int dd = tid; dd < kD; dd += nthr) {
    for (int h0 = 0; h0 < a.G; h0 += 2) {
      LseMerge mg[2];
      for (int p0 = 0; p0 < np; p0 += 4) {
        float2 ml[4][2];
        float ov[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int vp = p0 + i;
          const int slot = vp < n_seg ? vp : a.miss_base + (vp - n_seg);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = h0 + e;
            const bool on = vp < np && h < a.G;
            ml[i][e] = on ? __ldcg(&pml[slot * a.G + h]) : make_float2(-INFINITY, 0.f);
            ov[i][e] = on ? __ldcg(&po[((size_t)slot * a.G + h) * kD + dd]) : 0.f;
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

// A unit's output is ready once the hits pass has written one partial per
// segment (n_seg) and every fetched block its own (n_miss).  Each contributor
// calls this after writing its partial; the one that completes the count
// merges the unit, and the last unit merged ends the step (a.done_ctr).  No
// contributor waits for another.  tid / nthr: this thread among the threads
// that wrote the partial; sync(): a barrier over them; flag: one int of their
// shared memory.
template <class Sync>
__device__ void contribute_partial(const DecodeArgs& a, int u, int n_seg, int n_miss, int tid, int nthr,
                                   int* flag, Sync sync) {
  __threadfence();
  sync();
  if (tid == 0) *flag = (atomicAdd(&a.unit_done[u], 1) == n_seg + n_miss - 1);
  sync();
  if (*flag) {
    __threadfence();
    merge_unit(a, u, n_seg, n_miss, nullptr, tid, nthr);
    sync();
    if (tid == 0) {
      a.unit_done[u] = 0;
      if (a.done_ctr) {
        __threadfence();
        if (atomicAdd(a.done_ctr, 1) == a.U - 1) {
          __threadfence();
          advance_step(a.ds, a.st);
          *a.done_ctr = 0;
        }
      }
    }
  }
  sync();
}

// The hits pass walks a virtual sequence of positions: unit u owns positions
// [u * vpu, (u + 1) * vpu), vpu = k + tail_split + gap; position j < k of unit
// u is its j-th selected block (valid when j < k with KV resident, j <
// n_hit[u] otherwise), position k its open tail when tail_split is set (valid
// when it holds tokens), and the gap positions after them are never valid.
// CTA c takes the contiguous range [start(c), start(c + 1)), start(c) =
// floor(c * V / grid), so every CTA streams the same number of positions and
// touches one to a few units; each (unit, CTA) segment writes one partial.
// Ending a segment in mid-range (storing the partial, counting it, loading
// the next unit's queries) costs a CTA about as long as streaming a few
// blocks; the gap charges that time to the CTAs whose range crosses a unit
// boundary, which then stream fewer blocks.
struct Walk {
  long long V;
  int vpu, grid;
  __device__ long long start(int c) const { return (long long)c * V / grid; }
  // the CTA whose range holds position p
  __device__ int cta_of(long long p) const { return (int)(((p + 1) * grid - 1) / V); }
  __device__ int segments(int u) const {
    return cta_of((long long)(u + 1) * vpu - 1) - cta_of((long long)u * vpu) + 1;
  }
};

// Segments (partials) the hits pass writes for unit u, and the blocks fetched
// for it this step.
__device__ __forceinline__ int hits_segments(const DecodeArgs& a, int u) {
  Walk wk;
  wk.vpu = a.vpu;
  wk.V = (long long)a.U * wk.vpu;
  wk.grid = a.hits_grid;
  return wk.segments(u);
}
__device__ __forceinline__ int fetched_blocks(const DecodeArgs& a, int u) {
  return a.resident ? 0 : max(0, a.n_items[u] - a.n_hit[u]);
}

}  // namespace nosa
