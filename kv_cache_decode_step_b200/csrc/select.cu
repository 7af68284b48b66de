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
// Per unit and step t (S(-1) empty), F(t) = forced blocks (the first `sink`
// and last `window` closed blocks; App. B.2.2 counts them inside NOSA's
// query-agnostic budget):
//   Gamma_e(t) = top-(k_e - |F|) by agnostic score of Gamma_e(t-1) ∪ {blocks
//                that became eligible: closed outside the window or slid out}
//   c_t        = max(0, (k - m) - |(F ∪ Gamma_e)(t) \ S(t-1)|), unbounded at t = 0
//   Gamma_q(t) = top-k_q by score of (S(t-1) \ (F ∪ Gamma_e)) ∪ top-c_t(new)
//   S(t)       = F(t) ∪ Gamma_e(t) ∪ Gamma_q(t), ties to the lower block id.
//
// Lane l owns the blocks j with j % 32 == l.  Keys are order-preserving
// integer images of the scores (larger score -> larger key).  Up to 1024
// blocks the keys sit in registers and sets are per-lane bit masks, and a
// top-c set is found by a bitwise search over the keys (select_dev.cuh).
// Beyond that sets are bitmaps in shared memory (bit l of word j / 32), keys
// are read from memory, and one warp-wide argmax -- two redux.sync max steps,
// a ballot and, only on an exact tie, a redux.sync min over block ids --
// moves one block per round: choosing c of p candidates takes min(c, p - c)
// rounds, either moving the c best out or removing the p - c worst.
#include <climits>

#include "select_dev.cuh"

namespace nosa {

constexpr int kSelWarps = 4;
constexpr int kSmemKeys = 1024;  // query-aware keys staged in shared memory up to this many blocks

__device__ __forceinline__ unsigned valid_bits(int w, int n) {
  const int lo = w * 32;
  if (lo + 32 <= n) return kFull;
  if (lo >= n) return 0u;
  return (1u << (n - lo)) - 1u;
}

// Key source for a selection: staged 64-bit keys in shared memory, or the
// fp32 agnostic scores / fp64 scores in global memory.  `worst` flips the
// order (smallest score first, ties to the larger block id).
struct Keys {
  const unsigned long long* smem;
  const float* ag;
  const double* sc;
  bool worst;
  __device__ __forceinline__ unsigned long long raw(int j) const {
    if (smem) return smem[j];
    if (ag) return key_f32(ag[j]);
    return key_f64(sc[j]);
  }
  __device__ __forceinline__ unsigned long long operator()(int j) const {
    const unsigned long long k = raw(j);
    return worst ? ~k : k;
  }
  // tie order: smaller tie wins
  __device__ __forceinline__ unsigned tie(int j) const { return worst ? ~(unsigned)j : (unsigned)j; }
};

// This lane's best remaining candidate of `mask`.  Key 0 = none.
__device__ __forceinline__ void lane_best(const unsigned* mask, int words, int lane, const Keys& K,
                                          unsigned long long& bk, int& bj) {
  bk = 0ull;
  bj = -1;
  for (int w = 0; w < words; ++w) {
    if ((mask[w] >> lane) & 1u) {
      const int j = w * 32 + lane;
      const unsigned long long k = K(j);
      if (bj < 0 || k > bk || (k == bk && K.tie(j) < K.tie(bj))) {
        bk = k;
        bj = j;
      }
    }
  }
}

// Warp-wide winner of (key max, tie min); -1 when every lane is empty.
__device__ __forceinline__ int warp_winner(unsigned long long bk, int bj, const Keys& K, int lane) {
  const unsigned hi = (unsigned)(bk >> 32);
  const unsigned mhi = __reduce_max_sync(kFull, hi);
  if (mhi == 0u && __ballot_sync(kFull, bj >= 0) == 0u) return -1;
  const unsigned lo = (hi == mhi && bj >= 0) ? (unsigned)bk : 0u;
  const unsigned mlo = __reduce_max_sync(kFull, lo);
  const unsigned cand = __ballot_sync(kFull, bj >= 0 && hi == mhi && (unsigned)bk == mlo);
  if (__popc(cand) == 1) return __shfl_sync(kFull, bj, __ffs(cand) - 1);
  const unsigned t = ((cand >> lane) & 1u) ? K.tie(bj) : 0xffffffffu;
  const unsigned mt = __reduce_min_sync(kFull, t);
  const unsigned who = __ballot_sync(kFull, ((cand >> lane) & 1u) && t == mt);
  return __shfl_sync(kFull, bj, __ffs(who) - 1);
}

__device__ __forceinline__ int warp_popc(const unsigned* bm, int words, int lane) {
  int c = 0;
  for (int w = lane; w < words; w += 32) c += __popc(bm[w]);
  return __reduce_add_sync(kFull, c);
}

// Keep exactly the c best blocks of `mask` (in place).  Uses the cheaper of c
// argmax rounds into `tmp` or (p - c) argmin rounds out of `mask`.
__device__ void keep_best(unsigned* mask, unsigned* tmp, int words, int c, int lane, Keys K) {
  const int p = warp_popc(mask, words, lane);
  if (p <= c) return;
  const bool drop = (p - c) < c;
  K.worst = drop;
  const int rounds = drop ? p - c : c;
  if (!drop) {
    for (int w = lane; w < words; w += 32) tmp[w] = 0u;
    __syncwarp();
  }
  unsigned long long bk;
  int bj;
  lane_best(mask, words, lane, K, bk, bj);
  for (int r = 0; r < rounds; ++r) {
    const int j = warp_winner(bk, bj, K, lane);
    if (j < 0) break;
    if ((j & 31) == lane) {
      mask[j >> 5] &= ~(1u << lane);
      if (!drop) tmp[j >> 5] |= (1u << lane);
      lane_best(mask, words, lane, K, bk, bj);
    }
    __syncwarp();
  }
  if (!drop) {
    for (int w = lane; w < words; w += 32) mask[w] = tmp[w];
  }
  __syncwarp();
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

__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(SelectArgs a) {
  extern __shared__ unsigned long long sm_sel64[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kSelWarps + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.ds->gather_count = 0;
  if (u >= a.U) return;

  const int W = a.words;
  const bool stage = a.max_blocks <= kSmemKeys;
  unsigned long long* skeys = sm_sel64 + (size_t)warp * (stage ? a.max_blocks : 0);
  unsigned* bmE = reinterpret_cast<unsigned*>(sm_sel64 + (size_t)kSelWarps * (stage ? a.max_blocks : 0)) +
                  (size_t)warp * 4 * W;                 // Gamma_e(t)
  unsigned* bmP = bmE + W;                             // S(t-1)
  unsigned* bmX = bmP + W;                             // working set
  unsigned* bmT = bmX + W;                             // scratch / S(t)

  const int n = a.ds->n_closed;
  const int t = a.ds->step;
  const bool first = (t == 0);
  const int n_from = a.ds->n_last_select;
  const int nw = (n + 31) / 32;

  const double* sc = a.scores + (size_t)u * a.max_blocks;
  const float* ag = a.agnostic + (size_t)u * a.max_blocks;
  if (stage) {
    for (int j = lane; j < n; j += 32) skeys[j] = key_f64(sc[j]);
  }
  for (int w = lane; w < W; w += 32) {
    bmE[w] = 0u; bmP[w] = 0u; bmX[w] = 0u; bmT[w] = 0u;
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
      if (bj >= 0 && bj < n) atomicOr(&bmE[bj >> 5], 1u << (bj & 31));
    }
  }
  __syncwarp();

  // ---- Gamma_e over the eligible blocks [sink, n - window): unchanged
  // unless this is the first step or blocks became eligible since the last
  const Keys KA{nullptr, ag, nullptr, false};
  const Keys KS{stage ? skeys : nullptr, nullptr, sc, false};
  const int e_to = n - a.window;
  const int e_from = max(a.sink, first ? a.sink : n_from - a.window);
  if (e_from < e_to) {
    for (int w = lane; w < nw; w += 32) bmE[w] |= valid_bits(w, e_to) & ~valid_bits(w, e_from);
    __syncwarp();
    keep_best(bmE, bmT, nw, a.k_e - a.sink - a.window, lane, KA);
  }
  const int ne = bitmap_to_list(bmE, nw, ge, a.k_e, lane);
  for (int i = ne + lane; i < a.k_e; i += 32) ge[i] = -1;
  // from here on bmE holds F(t) ∪ Gamma_e(t): the sink and the window join it
  for (int w = lane; w < nw; w += 32)
    bmE[w] |= valid_bits(w, min(a.sink, n)) | (valid_bits(w, n) & ~valid_bits(w, max(0, n - a.window)));
  __syncwarp();

  // ---- Gamma_q
  if (first) {
    for (int w = lane; w < nw; w += 32) bmX[w] = valid_bits(w, n) & ~bmE[w];
    __syncwarp();
  } else {
    int e_new = 0;
    for (int w = lane; w < nw; w += 32) {
      e_new += __popc(bmE[w] & ~bmP[w]);
      bmX[w] = valid_bits(w, n) & ~bmE[w] & ~bmP[w];  // new candidates
    }
    e_new = __reduce_add_sync(kFull, e_new);
    const int c_t = max(0, a.c_max - e_new);
    __syncwarp();
    keep_best(bmX, bmT, nw, c_t, lane, KS);
    for (int w = lane; w < nw; w += 32) bmX[w] |= bmP[w] & ~bmE[w];  // ∪ old candidates
    __syncwarp();
  }
  keep_best(bmX, bmT, nw, a.k_q, lane, KS);

  int ov = 0;
  for (int w = lane; w < nw; w += 32) {
    bmX[w] |= bmE[w];  // S(t)
    ov += __popc(bmX[w] & bmP[w]);
  }
  ov = __reduce_add_sync(kFull, ov);
  __syncwarp();

  int* sel = a.sel + (size_t)u * a.k;
  const int ns = bitmap_to_list(bmX, nw, sel, a.k, lane);
  __syncwarp();
  for (int i = lane; i < a.k; i += 32) {
    const int v = i < ns ? sel[i] : -1;
    if (i >= ns) sel[i] = -1;
    prev[i] = v;
  }

  if (lane == 0) {
    atomicAdd(&a.st->selected, (unsigned long long)ns);
    if (!first) {
      atomicAdd(&a.st->overlap_sum, (unsigned long long)ov);
      atomicAdd(&a.st->overlap_terms, 1ull);
      atomicMin(&a.st->min_overlap, ov);
    }
  }
}

template <int R>
__global__ void __launch_bounds__(kSelWarps * 32) select_reg_kernel(SelectArgs a) {
  __shared__ unsigned sbm[kSelWarps][2][R];  // S(t-1) and Gamma_e(t-1) as block bitmaps
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kSelWarps + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.ds->gather_count = 0;
  if (u >= a.U) return;
  select_unit_reg<R>(a, u, lane, sbm[warp], a.scores + (size_t)u * a.max_blocks, a.prev + (size_t)u * a.k,
                     a.ge + (size_t)u * a.k_e, nullptr);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  const int grid = (a.U + kSelWarps - 1) / kSelWarps;
  // register path when every block fits in 32 rows per lane
  const int rows = (a.max_blocks + 31) / 32;
  if (rows <= 2) {
    select_reg_kernel<2><<<grid, kSelWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
  }
  if (rows <= 4) {
    select_reg_kernel<4><<<grid, kSelWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
  }
  if (rows <= 8) {
    select_reg_kernel<8><<<grid, kSelWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
  }
  if (rows <= 16) {
    select_reg_kernel<16><<<grid, kSelWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
  }
  if (rows <= 32) {
    select_reg_kernel<32><<<grid, kSelWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
  }
  const bool stage = a.max_blocks <= kSmemKeys;
  const size_t smem = (size_t)kSelWarps * ((stage ? a.max_blocks * sizeof(unsigned long long) : 0) +
                                           4 * a.words * sizeof(unsigned));
  select_kernel<<<grid, kSelWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nosa
