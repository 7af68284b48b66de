// plan_dev.cuh -- per-unit cache planning by one warp (set difference of the
// selection against the GPU block cache, replacement mapping, gather list),
// shared by the planning kernels and the fused score/select/plan kernel.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), §4 and
// App. A.  Replacement order: free slots (lowest first), then resident blocks
// outside S(t) by (last step selected, block id) ascending; the i-th miss
// (ascending block id) takes the i-th slot of that order.  A gather-list
// entry is (unit, block, slot, i): the block is the unit's i-th miss.
#pragma once

#include "nosa_internal.cuh"

namespace nosa {

constexpr unsigned kAll = 0xffffffffu;

// Plan of unit u by one warp, for any C and k.  The unit's slot tables are
// staged in shared memory (sm: 2 * C + 2 * k ints of this warp).  sel_in and
// bs_in: the unit's selection and block -> slot table (global memory, or
// copies in shared memory); staged: the slot tables already sit in sm.
__device__ __forceinline__ void plan_unit_smem(const PlanArgs& a, int u, int lane, int* sm, const int* sel_in,
                                               const int* bs_in, bool staged) {
  int* sb = sm;                                             // slot -> block
  int* lu = sb + a.C;                                       // slot -> last step selected
  int* smiss = lu + a.C;                                    // missed blocks, ascending
  int* ssrc = smiss + a.k;                                  // slots they will take

  const int t = a.ds->step;
  const int* sel = sel_in;
  int* slot_block = a.slot_block + (size_t)u * a.C;
  int* last_used = a.last_used + (size_t)u * a.C;
  int* block_slot = a.block_slot + (size_t)u * a.max_blocks;
  int* items = a.items + (size_t)u * a.k;
  const unsigned lt = (1u << lane) - 1u;

  if (!staged) {
    for (int c = lane; c < a.C; c += 32) {
      sb[c] = slot_block[c];
      lu[c] = last_used[c];
    }
    __syncwarp();
  }

  // 1. hits refresh their stamp; misses are listed in ascending order
  int n_hit = 0, n_miss = 0;
  for (int i0 = 0; i0 < a.k; i0 += 32) {
    const int i = i0 + lane;
    const int bj = i < a.k ? sel[i] : -1;
    const bool valid = bj >= 0 && bj < a.max_blocks;
    const int slot = valid ? bs_in[bj] : -1;
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
    int bc = -1;  // this lane's best candidate slot
    for (int c = lane; c < a.C; c += 32) {
      const int bj = sb[c];
      const int st = lu[c];
      if (bj >= 0 && st < t) {
        const unsigned h = (unsigned)st, l = (unsigned)bj;
        if (h < bhi || (h == bhi && l < blo)) {
          bhi = h;
          blo = l;
          bc = c;
        }
      }
    }
    const unsigned mhi = __reduce_min_sync(kAll, bhi);
    const unsigned mlo = __reduce_min_sync(kAll, bhi == mhi ? blo : 0xffffffffu);
    if (mhi == 0xffffffffu) {
      failed = true;
      break;
    }
    // slots hold distinct blocks: exactly one lane holds the winner's slot
    const unsigned win = __ballot_sync(kAll, bc >= 0 && bhi == mhi && blo == mlo);
    const int vslot = __shfl_sync(kAll, bc, __ffs(win) - 1);
    if (lane == 0) {
      ssrc[n_src] = vslot;
      block_slot[mlo] = -1;
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
      a.glist[base + i] = make_int4(u, bj, c, i);
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

// Plan of unit u by one warp for C <= 32 slots and k <= 32: lane s holds cache slot s and
// lane i holds the i-th selected block, so hits are found by matching the
// selection against the slot table with shuffles (no dependent global load)
// and the victim search is a pair of redux.sync minimums per victim.
// ssrc: 32 ints of this warp in shared memory; sel_in, sb_in, lu_in: the
// unit's selection, slot -> block and slot -> last-step tables (global memory,
// or copies in shared memory).
__device__ __forceinline__ void plan_unit_reg(const PlanArgs& a, int u, int lane, int* ssrc, const int* sel_in,
                                              const int* sb_in, const int* lu_in) {
  const int t = a.ds->step;
  int* slot_block = a.slot_block + (size_t)u * a.C;
  int* last_used = a.last_used + (size_t)u * a.C;
  int* block_slot = a.block_slot + (size_t)u * a.max_blocks;
  int* items = a.items + (size_t)u * a.k;
  const unsigned lt = (1u << lane) - 1u;

  const bool has_slot = lane < a.C;
  int sb = has_slot ? sb_in[lane] : -3;
  const int lu = has_slot ? lu_in[lane] : 0;
  const int bj = lane < a.k ? sel_in[lane] : -1;
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
  // reserve this unit's gather entries now; the round trip overlaps the rest
  int base = 0;
  if (lane == 0 && n_miss_all > 0) base = atomicAdd(&a.ds->gather_count, n_miss_all);
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
  base = __shfl_sync(kAll, base, 0);
  if (failed) {
    // no slot for the last misses: their reserved entries are marked invalid
    // (the gather skips them and flags a range error)
    if (lane == 0) atomicOr(&a.ds->error_bits, ERR_NOSLOT);
    n_miss = n_src;
    for (int i = n_miss + lane; i < n_miss_all; i += 32) a.glist[base + i] = make_int4(-1, -1, -1, 0);
  }

  // 4. install the misses (ascending block order) and emit the gather list
  const int mi = __popc(mm & lt);
  if (miss && mi < n_miss) {
    const int c = ssrc[mi];
    slot_block[c] = bj;
    last_used[c] = t;
    block_slot[bj] = c;
    items[n_hit + mi] = c;
    a.fetch[(size_t)u * a.k + mi] = bj;
    a.glist[base + mi] = make_int4(u, bj, c, mi);
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

}  // namespace nosa
