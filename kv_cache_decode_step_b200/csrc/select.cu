// select.cu -- locality-bounded block selection, one warp per unit.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary):
//   §2.1  query-aware top-k by query-key similarity; query-agnostic selection
//         scores units independently and keeps a fixed eviction pattern;
//   §3.1  the budget is divided between a query-aware and a query-agnostic
//         subset, with a minimum overlap gamma0 between adjacent steps;
//   App. E consecutive selections share at least k_e blocks.
// NOSA (gist.science explainer), technical summary, Method: a block dropped by
// the query-agnostic part is never taken back by it.
//
// Per unit and step t (S(-1) empty):
//   Gamma_e(t) = top-k_e by agnostic score of Gamma_e(t-1) ∪ {newly closed}
//   c_t        = max(0, (k - m) - |Gamma_e(t) \ S(t-1)|), unbounded at t = 0
//   Gamma_q(t) = top-k_q by score of (S(t-1) \ Gamma_e(t)) ∪ top-c_t(new)
//   S(t)       = Gamma_e(t) ∪ Gamma_q(t), ties to the lower block id.
// Sets are bitmaps in shared memory; lane l owns blocks j with j % 32 == l, so
// bit l of word i is block 32 i + l.  A top-c pass keeps each lane's best
// remaining candidate and, per round, reduces the warp's best with shuffles;
// only the winner's lane rescans its blocks.
#include <climits>

#include "nosa_internal.cuh"

namespace nosa {

constexpr int kSelWarps = 4;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ unsigned valid_bits(int w, int n) {
  const int lo = w * 32;
  if (lo + 32 <= n) return kFull;
  if (lo >= n) return 0u;
  return (1u << (n - lo)) - 1u;
}

// Better = larger key, then smaller id.
__device__ __forceinline__ bool better(double v, int i, double bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

template <typename KeyF>
__device__ __forceinline__ void lane_best(const unsigned* mask, int words, int lane, KeyF key, double& bv,
                                          int& bi) {
  bv = -INFINITY;
  bi = INT_MAX;
  for (int w = 0; w < words; ++w) {
    if ((mask[w] >> lane) & 1u) {
      const int j = w * 32 + lane;
      const double v = key(j);
      if (bi == INT_MAX || v > bv) {  // ascending j: equal keys keep the first
        bv = v;
        bi = j;
      }
    }
  }
}

// Move the `cnt` best blocks of `mask` into `out` (both bitmaps).
template <typename KeyF>
__device__ void warp_topk(unsigned* mask, unsigned* out, int words, int cnt, int lane, KeyF key) {
  if (cnt <= 0) return;
  double bv;
  int bi;
  lane_best(mask, words, lane, key, bv, bi);
  for (int r = 0; r < cnt; ++r) {
    double v = bv;
    int i = bi;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(kFull, v, o);
      const int oi = __shfl_xor_sync(kFull, i, o);
      if (oi != INT_MAX && (i == INT_MAX || better(ov, oi, v, i))) {
        v = ov;
        i = oi;
      }
    }
    if (i == INT_MAX) break;  // no candidates left (same on every lane)
    if ((i & 31) == lane) {
      mask[i >> 5] &= ~(1u << lane);
      out[i >> 5] |= (1u << lane);
      lane_best(mask, words, lane, key, bv, bi);
    }
    __syncwarp();
  }
}

// Write the set bits of bm in ascending order to out[0..cap); returns the count.
__device__ int bitmap_to_list(const unsigned* bm, int words, int* out, int cap, int lane) {
  int base = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    unsigned bits = w < words ? bm[w] : 0u;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += t;
    }
    int pos = base + incl - c;
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < cap) out[pos] = w * 32 + b;
      ++pos;
    }
    base += __shfl_sync(kFull, incl, 31);
  }
  return base;
}

__device__ __forceinline__ int warp_sum(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
  return x;
}

__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(SelectArgs a) {
  extern __shared__ unsigned sm_sel[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kSelWarps + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.ds->gather_count = 0;
  if (u >= a.U) return;

  const int W = a.words;
  unsigned* bmE = sm_sel + (size_t)warp * 4 * W;  // Gamma_e(t)
  unsigned* bmP = bmE + W;                         // S(t-1)
  unsigned* bmX = bmP + W;                         // working candidate set
  unsigned* bmS = bmX + W;                         // winners / S(t)

  const int n = a.ds->n_closed;
  const int t = a.ds->step;
  const bool first = (t == 0);
  const int n_from = a.ds->n_last_select;
  const int nw = (n + 31) / 32;

  for (int w = lane; w < W; w += 32) {
    bmE[w] = 0u; bmP[w] = 0u; bmX[w] = 0u; bmS[w] = 0u;
  }
  __syncwarp();

  int* prev = a.prev + (size_t)u * a.k;
  int* ge = a.ge + (size_t)u * a.k_e;
  if (!first) {
    for (int i = lane; i < a.k; i += 32) {
      const int bj = prev[i];
      if (bj >= 0 && bj < n) atomicOr(&bmP[bj >> 5], 1u << (bj & 31));
    }
    for (int i = lane; i < a.k_e; i += 32) {
      const int bj = ge[i];
      if (bj >= 0 && bj < n) atomicOr(&bmX[bj >> 5], 1u << (bj & 31));
    }
  }
  __syncwarp();
  // pool of Gamma_e: everything at t = 0, else Gamma_e(t-1) ∪ [n_from, n)
  const int pool_lo = first ? 0 : n_from;
  for (int w = lane; w < nw; w += 32) {
    unsigned add = valid_bits(w, n) & ~valid_bits(w, pool_lo);
    bmX[w] |= add;
  }
  __syncwarp();

  const float* ag = a.agnostic + (size_t)u * a.max_blocks;
  const double* sc = a.scores + (size_t)u * a.max_blocks;
  auto key_a = [ag](int j) { return (double)ag[j]; };
  auto key_s = [sc](int j) { return sc[j]; };

  warp_topk(bmX, bmE, nw, a.k_e, lane, key_a);
  __syncwarp();

  if (first) {
    for (int w = lane; w < nw; w += 32) bmX[w] = valid_bits(w, n) & ~bmE[w];
  } else {
    int e_new = 0;
    for (int w = lane; w < nw; w += 32) {
      e_new += __popc(bmE[w] & ~bmP[w]);
      bmX[w] = valid_bits(w, n) & ~bmE[w] & ~bmP[w];  // new candidates
    }
    e_new = warp_sum(e_new);
    const int c_t = max(0, a.c_max - e_new);
    __syncwarp();
    warp_topk(bmX, bmS, nw, c_t, lane, key_s);
    __syncwarp();
    for (int w = lane; w < nw; w += 32) {
      bmX[w] = (bmP[w] & ~bmE[w]) | bmS[w];
      bmS[w] = 0u;
    }
  }
  __syncwarp();
  warp_topk(bmX, bmS, nw, a.k_q, lane, key_s);
  __syncwarp();

  int ov = 0;
  for (int w = lane; w < nw; w += 32) {
    bmS[w] |= bmE[w];
    ov += __popc(bmS[w] & bmP[w]);
  }
  ov = warp_sum(ov);
  __syncwarp();

  int* sel = a.sel + (size_t)u * a.k;
  const int ns = bitmap_to_list(bmS, nw, sel, a.k, lane);
  __syncwarp();
  for (int i = lane; i < a.k; i += 32) {
    const int v = i < ns ? sel[i] : -1;
    if (i >= ns) sel[i] = -1;
    prev[i] = v;
  }
  const int ne = bitmap_to_list(bmE, nw, ge, a.k_e, lane);
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

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  const int grid = (a.U + kSelWarps - 1) / kSelWarps;
  const size_t smem = (size_t)kSelWarps * 4 * a.words * sizeof(unsigned);
  select_kernel<<<grid, kSelWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nosa
