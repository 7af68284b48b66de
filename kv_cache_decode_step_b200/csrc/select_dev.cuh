// select_dev.cuh -- per-unit selection by one warp with keys in registers,
// shared by the selection kernel and the fused score/select/plan kernel.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), §2.1,
// §3.1, App. B.2.2 and App. E; the rule itself is stated in select.cu.
#pragma once

#include "nosa_internal.cuh"

namespace nosa {

constexpr unsigned kFull = 0xffffffffu;

// Order-preserving maps to unsigned integers.  No real key maps to 0, which
// marks "no candidate".  -0.0 and +0.0 compare equal, so both map to the key
// of +0.0 and their order falls to the block ids like any other tie.
__device__ __forceinline__ unsigned long long key_f64(double x) {
  if (x == 0.0) x = 0.0;
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  return (b & 0x8000000000000000ull) ? ~b : (b | 0x8000000000000000ull);
}
__device__ __forceinline__ unsigned long long key_f32(float x) {
  if (x == 0.0f) x = 0.0f;
  const unsigned b = __float_as_uint(x);
  return (unsigned long long)((b & 0x80000000u) ? ~b : (b | 0x80000000u)) << 32;
}

// ---------------------------------------------------------------- register path
// For n <= 32 * R: lane l holds blocks j = 32 i + l (i < R) -- their keys in
// registers and set membership as R-bit masks -- so choosing a top-c set is a
// bitwise search with one warp-wide count per key bit, and lists come out of
// one ballot per row i.

// Keep exactly the c best of `mask` (per-lane R-bit masks, whole warp): the
// c largest keys, the lower block id first among equal keys.  Radix
// selection: the threshold key is fixed one bit at a time, most significant
// first; `cand` holds the members that still agree with the threshold's
// prefix, `kept` those already above it.  Each bit costs one warp-wide count
// (redux.sync), and the search stops as soon as the candidates left are
// exactly the ones still needed.  Members whose whole key equals the
// threshold are then told apart the same way on their block ids
// j = 32 i + lane (smaller ids first).
template <int R>
__device__ __forceinline__ void keep_best_reg(uint32_t& mask, int c, const unsigned long long (&k)[R], int lane) {
  int left = (int)__reduce_add_sync(kFull, (unsigned)__popc(mask));  // members in cand
  if (left <= c) return;
  uint32_t kept = 0u, cand = mask;
  int need = c;
  // Key bits on which all members agree split nothing (every member goes the
  // same way): the search starts at the highest bit where two members differ.
  unsigned long long k_and = ~0ull, k_or = 0ull;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if ((mask >> i) & 1u) {
      k_and &= k[i];
      k_or |= k[i];
    }
  }
  const unsigned d_hi = __reduce_or_sync(kFull, (unsigned)(k_or >> 32)) & ~__reduce_and_sync(kFull, (unsigned)(k_and >> 32));
  const unsigned d_lo = __reduce_or_sync(kFull, (unsigned)k_or) & ~__reduce_and_sync(kFull, (unsigned)k_and);
  const int b_top = d_hi ? 63 - __clz(d_hi) : (d_lo ? 31 - __clz(d_lo) : -1);
  // 64 key bits: the high words, then the low words
#pragma unroll 1
  for (int b = b_top; b >= 0 && need > 0 && need < left; --b) {
    uint32_t ones = 0u;
#pragma unroll
    for (int i = 0; i < R; ++i) ones |= (uint32_t)((k[i] >> b) & 1ull) << i;
    ones &= cand;
    const int n1 = (int)__reduce_add_sync(kFull, (unsigned)__popc(ones));
    if (n1 >= need) {  // the threshold has this bit set: members without it fall out
      cand = ones;
      left = n1;
    } else {           // it has this bit clear: members with it are above the threshold
      kept |= ones;
      need -= n1;
      cand &= ~ones;
      left -= n1;
    }
  }
  // equal keys: the smaller block ids (bits 5.. of j are the row i, bits 0..4 the lane)
#pragma unroll 1
  for (int b = 9; b >= 0 && need > 0 && need < left; --b) {
    uint32_t zeros = 0u;
    if (b >= 5) {
#pragma unroll
      for (int i = 0; i < R; ++i) zeros |= (((i >> (b - 5)) & 1) ? 0u : 1u) << i;
    } else {
      zeros = ((lane >> b) & 1) ? 0u : 0xffffffffu;
    }
    zeros &= cand;
    const int n0 = (int)__reduce_add_sync(kFull, (unsigned)__popc(zeros));
    if (n0 >= need) {
      cand = zeros;
      left = n0;
    } else {
      kept |= zeros;
      need -= n0;
      cand &= ~zeros;
      left -= n0;
    }
  }
  if (need > 0) kept |= cand;  // need == left: every candidate left is in
  mask = kept;
}

// Blocks of the per-lane masks, ascending, into out[0..cap) and, when given,
// into out2 and out3 as well (one walk over the rows); returns the count.
// Up to 8 rows per lane all R ballots are taken first (they do not depend on
// one another) and the positions follow from their running counts; with more
// rows, one row at a time (fewer registers live).
template <int R>
__device__ __forceinline__ int write_list_reg(uint32_t mask, int* out, int cap, int lane, int* out2 = nullptr,
                                              int* out3 = nullptr) {
  const unsigned lt = (1u << lane) - 1u;
  int base = 0;
  if constexpr (R <= 8) {
    unsigned bal[R];
#pragma unroll
    for (int i = 0; i < R; ++i) bal[i] = __ballot_sync(kFull, (mask >> i) & 1u);
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int pos = base + __popc(bal[i] & lt);
      if (((mask >> i) & 1u) && pos < cap) {
        const int j = 32 * i + lane;
        out[pos] = j;
        if (out2) out2[pos] = j;
        if (out3) out3[pos] = j;
      }
      base += __popc(bal[i]);
    }
  } else {
#pragma unroll 4
    for (int i = 0; i < R; ++i) {
      const bool on = (mask >> i) & 1u;
      const unsigned bal = __ballot_sync(kFull, on);
      const int pos = base + __popc(bal & lt);
      if (on && pos < cap) {
        const int j = 32 * i + lane;
        out[pos] = j;
        if (out2) out2[pos] = j;
        if (out3) out3[pos] = j;
      }
      base += __popc(bal);
    }
  }
  return base;
}

// Selection of unit u by one warp (lane = lane id), keys in registers: every
// closed block must satisfy j < 32 * R.  sc: the unit's fp64 scores; prev_in,
// ge_in: the unit's S(t-1) and Gamma_e(t-1) (global memory, or a copy in
// shared memory); sbm: per-warp scratch of 2 x R words in shared memory;
// sel_copy: null, or k ints that also receive the selection.
template <int R>
__device__ __forceinline__ void select_unit_reg(const SelectArgs& a, int u, int lane, unsigned (*sbm)[R],
                                                const double* sc, const int* prev_in, const int* ge_in,
                                                int* sel_copy) {
  const int n = a.ds->n_closed;
  const int t = a.ds->step;
  const bool first = (t == 0);
  const int n_from = a.ds->n_last_select;
  const float* ag = a.agnostic + (size_t)u * a.max_blocks;
  int* prev = a.prev + (size_t)u * a.k;
  int* ge = a.ge + (size_t)u * a.k_e;

  unsigned long long ks[R];
  // closed blocks; blocks that became eligible for Gamma_e since the last
  // step ([sink, n - window) minus what was eligible then); forced blocks
  uint32_t valid = 0u, fresh = 0u, forced = 0u;
  const int e_to = n - a.window;
  const int e_from = max(a.sink, first ? a.sink : n_from - a.window);
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int j = 32 * i + lane;
    ks[i] = j < n ? key_f64(sc[j]) : 0ull;
    if (j < n) valid |= 1u << i;
    if (j >= e_from && j < e_to) fresh |= 1u << i;
    if (j < n && (j < a.sink || j >= n - a.window)) forced |= 1u << i;
  }
  for (int i = lane; i < 2 * R; i += 32) (&sbm[0][0])[i] = 0u;
  __syncwarp();
  if (!first) {
    for (int i = lane; i < a.k; i += 32) {
      const int bj = prev_in[i];
      if (bj >= 0 && bj < n) atomicOr(&sbm[0][bj >> 5], 1u << (bj & 31));
    }
    for (int i = lane; i < a.k_e; i += 32) {
      const int bj = ge_in[i];
      if (bj >= 0 && bj < n) atomicOr(&sbm[1][bj >> 5], 1u << (bj & 31));
    }
  }
  __syncwarp();
  uint32_t mP = 0u, mE = 0u;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    mP |= ((sbm[0][i] >> lane) & 1u) << i;
    mE |= ((sbm[1][i] >> lane) & 1u) << i;
  }

  // ---- Gamma_e over the eligible blocks: unchanged unless this is the first
  // step or blocks became eligible since the last
  if (__any_sync(kFull, fresh != 0u)) {
    unsigned long long ka[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int j = 32 * i + lane;
      ka[i] = j < n ? key_f32(ag[j]) : 0ull;
    }
    mE |= fresh;
    keep_best_reg<R>(mE, a.k_e - a.sink - a.window, ka, lane);
  }

  // ---- Gamma_q, outside F(t) ∪ Gamma_e(t)
  const uint32_t mF = mE | forced;
  uint32_t mX;
  if (first) {
    mX = valid & ~mF;
  } else {
    const int e_new = (int)__reduce_add_sync(kFull, (unsigned)__popc(mF & ~mP));
    const int c_t = max(0, a.c_max - e_new);
    mX = valid & ~mF & ~mP;  // new candidates
    keep_best_reg<R>(mX, c_t, ks, lane);
    mX |= mP & ~mF;          // ∪ old candidates
  }
  keep_best_reg<R>(mX, a.k_q, ks, lane);
  const uint32_t mS = mX | mF;
  const int ov = (int)__reduce_add_sync(kFull, (unsigned)__popc(mS & mP));

  int* sel = a.sel + (size_t)u * a.k;
  const int ns = write_list_reg<R>(mS, sel, a.k, lane, prev, sel_copy);
  for (int i = ns + lane; i < a.k; i += 32) {
    sel[i] = -1;
    prev[i] = -1;
    if (sel_copy) sel_copy[i] = -1;
  }
  const int ne = write_list_reg<R>(mE, ge, a.k_e, lane);
  for (int i = ne + lane; i < a.k_e; i += 32) ge[i] = -1;

  if (lane == 0) {
    atomicAdd(&a.st->selected, (unsigned long long)ns);
    if (!first) {
      atomicAdd(&a.st->overlap_sum, (unsigned long long)ov);
      atomicAdd(&a.st->overlap_terms, 1ull);
      atomicMin(&a.st->min_overlap, ov);
    }
  }
}

// ---------------------------------------------------------------- group path
// W warps of one CTA select one unit together: warp w holds rows
// [w*RW, (w+1)*RW) of the register layout, i.e. blocks j = 32 (w RW + i) +
// lane for i < RW, so each lane has RW keys instead of W*RW.  Every count and
// bitwise reduction of the one-warp path becomes a warp reduction, a word per
// warp in shared memory and one named barrier over the W warps; the search
// takes the same steps on the same totals, so the selection is the same.

// Shared-memory reductions over the W warps.  red: [2][W][4] words; phase
// alternates the two halves, so a warp that runs ahead never overwrites a
// word another warp has still to read (a barrier separates any two uses of
// one half).  Every warp of the group must make the same sequence of calls.
template <int W>
struct SelGroup {
  unsigned* red;
  int w, lane, bar;
  int phase = 0;
  __device__ void sync() const { bar_sync(bar, W * 32); }
  __device__ unsigned* slot() { unsigned* r = red + (phase & 1) * W * 4; ++phase; return r; }
  // sum of x over the group (x is per lane)
  __device__ int sum(int x) {
    const unsigned s = __reduce_add_sync(kFull, (unsigned)x);
    unsigned* r = slot();
    if (lane == 0) r[w * 4] = s;
    sync();
    unsigned t = 0;
#pragma unroll
    for (int v = 0; v < W; ++v) t += r[v * 4];
    return (int)t;
  }
  // exclusive prefix over warps of a per-warp count x (equal in all lanes);
  // *total receives the group's sum
  __device__ int prefix(int x, int* total) {
    unsigned* r = slot();
    if (lane == 0) r[w * 4] = (unsigned)x;
    sync();
    int before = 0, all = 0;
#pragma unroll
    for (int v = 0; v < W; ++v) {
      const int c = (int)r[v * 4];
      if (v < w) before += c;
      all += c;
    }
    *total = all;
    return before;
  }
  // group-wide OR of o and AND of a, each a 64-bit per-lane value
  __device__ void or_and(unsigned long long& o, unsigned long long& a) {
    const unsigned oh = __reduce_or_sync(kFull, (unsigned)(o >> 32)), ol = __reduce_or_sync(kFull, (unsigned)o);
    const unsigned ah = __reduce_and_sync(kFull, (unsigned)(a >> 32)), al = __reduce_and_sync(kFull, (unsigned)a);
    unsigned* r = slot();
    if (lane == 0) {
      r[w * 4 + 0] = oh;
      r[w * 4 + 1] = ol;
      r[w * 4 + 2] = ah;
      r[w * 4 + 3] = al;
    }
    sync();
    unsigned toh = 0u, tol = 0u, tah = ~0u, tal = ~0u;
#pragma unroll
    for (int v = 0; v < W; ++v) {
      toh |= r[v * 4 + 0];
      tol |= r[v * 4 + 1];
      tah &= r[v * 4 + 2];
      tal &= r[v * 4 + 3];
    }
    o = ((unsigned long long)toh << 32) | tol;
    a = ((unsigned long long)tah << 32) | tal;
  }
};

// keep_best_reg over the group: the same radix search on group-wide counts.
template <int RW, int W>
__device__ __forceinline__ void keep_best_group(uint32_t& mask, int c, const unsigned long long (&k)[RW],
                                                SelGroup<W>& g) {
  int left = g.sum(__popc(mask));
  if (left <= c) return;
  uint32_t kept = 0u, cand = mask;
  int need = c;
  unsigned long long k_and = ~0ull, k_or = 0ull;
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    if ((mask >> i) & 1u) {
      k_and &= k[i];
      k_or |= k[i];
    }
  }
  g.or_and(k_or, k_and);
  const unsigned long long diff = k_or & ~k_and;
  const int b_top = diff ? 63 - __clzll((long long)diff) : -1;
#pragma unroll 1
  for (int b = b_top; b >= 0 && need > 0 && need < left; --b) {
    uint32_t ones = 0u;
#pragma unroll
    for (int i = 0; i < RW; ++i) ones |= (uint32_t)((k[i] >> b) & 1ull) << i;
    ones &= cand;
    const int n1 = g.sum(__popc(ones));
    if (n1 >= need) {
      cand = ones;
      left = n1;
    } else {
      kept |= ones;
      need -= n1;
      cand &= ~ones;
      left -= n1;
    }
  }
  // equal keys: the smaller block ids (bits 5.. of j are the row w RW + i)
#pragma unroll 1
  for (int b = 9; b >= 0 && need > 0 && need < left; --b) {
    uint32_t zeros = 0u;
    if (b >= 5) {
#pragma unroll
      for (int i = 0; i < RW; ++i) zeros |= ((((g.w * RW + i) >> (b - 5)) & 1) ? 0u : 1u) << i;
    } else {
      zeros = ((g.lane >> b) & 1) ? 0u : 0xffffffffu;
    }
    zeros &= cand;
    const int n0 = g.sum(__popc(zeros));
    if (n0 >= need) {
      cand = zeros;
      left = n0;
    } else {
      kept |= zeros;
      need -= n0;
      cand &= ~zeros;
      left -= n0;
    }
  }
  if (need > 0) kept |= cand;
  mask = kept;
}

// write_list_reg over the group: warp w's blocks follow those of warps < w.
template <int RW, int W>
__device__ __forceinline__ int write_list_group(uint32_t mask, int* out, int cap, SelGroup<W>& g,
                                                int* out2 = nullptr, int* out3 = nullptr) {
  const unsigned lt = (1u << g.lane) - 1u;
  unsigned bal[RW];
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    bal[i] = __ballot_sync(kFull, (mask >> i) & 1u);
    cnt += __popc(bal[i]);
  }
  int total = 0;
  int base = g.prefix(cnt, &total);
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    const int pos = base + __popc(bal[i] & lt);
    if (((mask >> i) & 1u) && pos < cap) {
      const int j = 32 * (g.w * RW + i) + g.lane;
      out[pos] = j;
      if (out2) out2[pos] = j;
      if (out3) out3[pos] = j;
    }
    base += __popc(bal[i]);
  }
  return total;
}

// select_unit_reg by W warps (see the group path above): every closed block
// must satisfy j < 32 * W * RW.  sbm: 2 x (W * RW) words of shared memory for
// the group; sc, prev_in, ge_in, sel_copy as for select_unit_reg.
template <int RW, int W>
__device__ __forceinline__ void select_unit_group(const SelectArgs& a, int u, SelGroup<W>& g, unsigned* sbm,
                                                  const double* sc, const int* prev_in, const int* ge_in,
                                                  int* sel_copy) {
  constexpr int R = RW * W;
  const int lane = g.lane, row0 = g.w * RW, tid = g.w * 32 + lane;
  const int n = a.ds->n_closed;
  const int t = a.ds->step;
  const bool first = (t == 0);
  const int n_from = a.ds->n_last_select;
  const float* ag = a.agnostic + (size_t)u * a.max_blocks;
  int* prev = a.prev + (size_t)u * a.k;
  int* ge = a.ge + (size_t)u * a.k_e;

  unsigned long long ks[RW];
  uint32_t valid = 0u, fresh = 0u, forced = 0u;
  const int e_to = n - a.window;
  const int e_from = max(a.sink, first ? a.sink : n_from - a.window);
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    const int j = 32 * (row0 + i) + lane;
    ks[i] = j < n ? key_f64(sc[j]) : 0ull;
    if (j < n) valid |= 1u << i;
    if (j >= e_from && j < e_to) fresh |= 1u << i;
    if (j < n && (j < a.sink || j >= n - a.window)) forced |= 1u << i;
  }
  for (int i = tid; i < 2 * R; i += W * 32) sbm[i] = 0u;
  g.sync();
  if (!first) {
    for (int i = tid; i < a.k; i += W * 32) {
      const int bj = prev_in[i];
      if (bj >= 0 && bj < n) atomicOr(&sbm[bj >> 5], 1u << (bj & 31));
    }
    for (int i = tid; i < a.k_e; i += W * 32) {
      const int bj = ge_in[i];
      if (bj >= 0 && bj < n) atomicOr(&sbm[R + (bj >> 5)], 1u << (bj & 31));
    }
  }
  g.sync();
  uint32_t mP = 0u, mE = 0u;
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    mP |= ((sbm[row0 + i] >> lane) & 1u) << i;
    mE |= ((sbm[R + row0 + i] >> lane) & 1u) << i;
  }

  if (g.sum(__any_sync(kFull, fresh != 0u) ? 1 : 0) > 0) {
    unsigned long long ka[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      const int j = 32 * (row0 + i) + lane;
      ka[i] = j < n ? key_f32(ag[j]) : 0ull;
    }
    mE |= fresh;
    keep_best_group<RW, W>(mE, a.k_e - a.sink - a.window, ka, g);
  }

  const uint32_t mF = mE | forced;
  uint32_t mX;
  if (first) {
    mX = valid & ~mF;
  } else {
    const int e_new = g.sum(__popc(mF & ~mP));
    const int c_t = max(0, a.c_max - e_new);
    mX = valid & ~mF & ~mP;
    keep_best_group<RW, W>(mX, c_t, ks, g);
    mX |= mP & ~mF;
  }
  keep_best_group<RW, W>(mX, a.k_q, ks, g);
  const uint32_t mS = mX | mF;
  const int ov = g.sum(__popc(mS & mP));

  int* sel = a.sel + (size_t)u * a.k;
  const int ns = write_list_group<RW, W>(mS, sel, a.k, g, prev, sel_copy);
  for (int i = ns + tid; i < a.k; i += W * 32) {
    sel[i] = -1;
    prev[i] = -1;
    if (sel_copy) sel_copy[i] = -1;
  }
  const int ne = write_list_group<RW, W>(mE, ge, a.k_e, g);
  for (int i = ne + tid; i < a.k_e; i += W * 32) ge[i] = -1;

  if (tid == 0) {
    atomicAdd(&a.st->selected, (unsigned long long)ns);
    if (!first) {
      atomicAdd(&a.st->overlap_sum, (unsigned long long)ov);
      atomicAdd(&a.st->overlap_terms, 1ull);
      atomicMin(&a.st->min_overlap, ov);
    }
  }
}

}  // namespace nosa
