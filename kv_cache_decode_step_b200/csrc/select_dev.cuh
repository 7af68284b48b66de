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
// marks "no candidate".
__device__ __forceinline__ unsigned long long key_f64(double x) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  return (b & 0x8000000000000000ull) ? ~b : (b | 0x8000000000000000ull);
}
__device__ __forceinline__ unsigned long long key_f32(float x) {
  const unsigned b = __float_as_uint(x);
  return (unsigned long long)((b & 0x80000000u) ? ~b : (b | 0x80000000u)) << 32;
}

// ---------------------------------------------------------------- register path
// For n <= 32 * R: lane l holds blocks j = 32 i + l (i < R) -- their keys in
// registers and set membership as R-bit masks -- so a round of selection is a
// warp_winner plus an R-step rescan in registers, and lists come out of one
// ballot per row i.

template <int R>
__device__ __forceinline__ void lane_best_reg(uint32_t mask, const unsigned long long (&k)[R], bool worst,
                                              unsigned long long& bk, int& bi) {
  bk = 0ull;
  bi = -1;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if ((mask >> i) & 1u) {
      const unsigned long long kk = worst ? ~k[i] : k[i];
      // rows ascend with i: on equal keys keep the first for "best", the last for "worst"
      if (bi < 0 || kk > bk || (worst && kk == bk)) {
        bk = kk;
        bi = i;
      }
    }
  }
}

// Keep exactly the c best of `mask` (per-lane R-bit masks, whole warp).
template <int R>
__device__ void keep_best_reg(uint32_t& mask, int c, const unsigned long long (&k)[R], int lane) {
  const int p = (int)__reduce_add_sync(kFull, (unsigned)__popc(mask));
  if (p <= c) return;
  const bool worst = (p - c) < c;
  const int rounds = worst ? p - c : c;
  uint32_t kept = 0u;
  unsigned long long bk;
  int bi;
  lane_best_reg<R>(mask, k, worst, bk, bi);
  for (int r = 0; r < rounds; ++r) {
    const unsigned hi = (unsigned)(bk >> 32);
    const unsigned mhi = __reduce_max_sync(kFull, hi);
    if (mhi == 0u) break;
    const unsigned lo = (bi >= 0 && hi == mhi) ? (unsigned)bk : 0u;
    const unsigned mlo = __reduce_max_sync(kFull, lo);
    const unsigned cand = __ballot_sync(kFull, bi >= 0 && hi == mhi && (unsigned)bk == mlo);
    int wl;  // winning lane
    if (__popc(cand) == 1) {
      wl = __ffs(cand) - 1;
    } else {
      // equal keys: block id 32*bi + lane decides (smaller for best, larger for worst)
      const unsigned j = (unsigned)(32 * bi + lane);
      const unsigned t = ((cand >> lane) & 1u) ? (worst ? ~j : j) : 0xffffffffu;
      const unsigned mt = __reduce_min_sync(kFull, t);
      wl = __ffs(__ballot_sync(kFull, ((cand >> lane) & 1u) && t == mt)) - 1;
    }
    if (lane == wl) {
      mask &= ~(1u << bi);
      if (!worst) kept |= 1u << bi;
      lane_best_reg<R>(mask, k, worst, bk, bi);
    }
  }
  if (!worst) mask = kept;
}

// Blocks of the per-lane masks, ascending, into out[0..cap); returns the count.
template <int R>
__device__ __forceinline__ int write_list_reg(uint32_t mask, int* out, int cap, int lane) {
  const unsigned lt = (1u << lane) - 1u;
  int base = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const bool on = (mask >> i) & 1u;
    const unsigned bal = __ballot_sync(kFull, on);
    const int pos = base + __popc(bal & lt);
    if (on && pos < cap) out[pos] = 32 * i + lane;
    base += __popc(bal);
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
  const int ns = write_list_reg<R>(mS, sel, a.k, lane);
  write_list_reg<R>(mS, prev, a.k, lane);
  if (sel_copy) write_list_reg<R>(mS, sel_copy, a.k, lane);
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

}  // namespace nosa
