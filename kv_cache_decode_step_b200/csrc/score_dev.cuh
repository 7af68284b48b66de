// score_dev.cuh -- block scoring helpers shared by the scoring kernel and
// the fused score/select/plan kernel.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), §3.1:
// a block's score is the largest of its sub-blocks' scores, each the
// group-summed query against the sub-block's mean-pooled key.  Lane 8r + c of
// a warp holds sub-block r of a block and owns dims [8c, 8c+8) and
// [64+8c, 64+8c+8); the group's queries are summed first (fp64, exact for
// bf16 inputs), so each sub-block score is one 128-term fp64 dot product
// whose products are exact.
#pragma once

#include <type_traits>

#include "nosa_internal.cuh"

namespace nosa {

constexpr int kBlockU4 = kR * kRowU4;  // 16-byte words of pooled keys per block (64)

// One 16-byte word's contribution (dims 2i .. 2i+7 of qt), fma by fma.  With
// kPlaced the upper bf16 of each 32-bit word is widened by bit placement
// (bf16_hi_placed_f64) and its query term qt[2i+1] is expected scaled by
// 2^896: the fp64 pipe, which also runs the conversions, then widens only
// half of the keys, the other half goes to the integer pipe, and every fma
// rounds exactly as with two conversions.
template <bool kPlaced>
__device__ __forceinline__ double dot8_acc(const uint4& a, const double* qt, double s) {
  const uint32_t wv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s = fma(qt[2 * i], bf16_lo_to_f64(wv[i]), s);
    s = fma(qt[2 * i + 1], kPlaced ? bf16_hi_placed_f64(wv[i]) : bf16_hi_to_f64(wv[i]), s);
  }
  return s;
}

template <bool kPlaced>
__device__ __forceinline__ double dot16(const uint4& a, const uint4& b, const double* qt) {
  return dot8_acc<kPlaced>(b, qt + 8, dot8_acc<kPlaced>(a, qt, 0.0));
}

// Whether this warp may use placed widening: every lane's odd query sums,
// scaled by 2^896, stay finite (|qt| < 2^126 leaves a margin).  If so, they
// are scaled in place.  Warp-wide vote: both paths give the same bits.
__device__ __forceinline__ bool place_query_terms(double (&qt)[16]) {
  bool ok = true;
#pragma unroll
  for (int i = 1; i < 16; i += 2) ok = ok && fabs(qt[i]) < 0x1p126;
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
#pragma unroll
    for (int i = 1; i < 16; i += 2) qt[i] *= kBf16PlaceScale;
  }
  return ok;
}

// Scores of NB blocks (NB = 4 or 8) from this lane's partial sums s[i] of
// block i: the sum over the 8 lanes of each sub-block, then the max over the
// 4 sub-blocks.  The sums halve the values per lane at each step: across
// lanes l and l ^ d a lane keeps the blocks whose index bit matches its own
// lane bit and sends the others to its partner, so after the steps d = 1, 2, 4
// lane 8r + c holds sub-block r's sum of block c % NB.  Every sum pairs the
// same operands as a butterfly over each block in turn, so the results are
// the same bits.  Lanes c % NB = i return block i's score.
template <int NB>
__device__ __forceinline__ double blocks_reduce(const double (&s)[NB], int lane) {
  static_assert(NB == 4 || NB == 8, "4 or 8 blocks");
  double v[NB];
#pragma unroll
  for (int i = 0; i < NB; ++i) v[i] = s[i];
  int m = NB;
#pragma unroll
  for (int d = 1; d < 8; d <<= 1) {
    if (m > 1) {
      const bool odd = (lane & d) != 0;
#pragma unroll
      for (int i = 0; i < NB / 2; ++i) {
        if (i < m / 2) {
          const double keep = odd ? v[2 * i + 1] : v[2 * i];
          const double send = odd ? v[2 * i] : v[2 * i + 1];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, d);
        }
      }
      m /= 2;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], d);
    }
  }
  double o = __shfl_xor_sync(0xffffffffu, v[0], 8);
  double x = o > v[0] ? o : v[0];
  o = __shfl_xor_sync(0xffffffffu, x, 16);
  return o > x ? o : x;
}

// qt = sum over the unit's G query heads of their dims [8c, 8c+8) and
// [64+8c, 64+8c+8), in fp64.  q_rows: the unit's G query rows (shared
// memory), or null to read them from a.q.
__device__ __forceinline__ void group_query_sum(const ScoreArgs& a, int b, int g, int c, double (&qt)[16],
                                                const uint4* q_rows = nullptr) {
#pragma unroll
  for (int i = 0; i < 16; ++i) qt[i] = 0.0;
  const uint4* qrow =
      q_rows ? q_rows : reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + (size_t)g * a.G) * kD);
  for (int h = 0; h < a.G; ++h) {
    const uint4 y0 = qrow[h * kRowU4 + c], y1 = qrow[h * kRowU4 + 8 + c];
    const uint32_t wv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qt[2 * i] += bf16_lo_to_f64(wv[i]);
      qt[2 * i + 1] += bf16_hi_to_f64(wv[i]);
    }
  }
}

// Scores of groups of 4 consecutive blocks: loads into (x, y), then dot
// products, reductions and the stores of the group's scores.
__device__ __forceinline__ void score_group_load(const uint4* base, int g0, int cnt, int c, uint4 (&x)[4],
                                                 uint4 (&y)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i < cnt) {
      const uint4* row = base + (size_t)(g0 + i) * kBlockU4;
      x[i] = __ldg(row + c);
      y[i] = __ldg(row + 8 + c);
    }
  }
}

template <bool kPlaced>
__device__ __forceinline__ void score_group_finish(const ScoreArgs& a, int u, int g0, int cnt, int lane,
                                                   const uint4 (&x)[4], const uint4 (&y)[4], const double (&qt)[16],
                                                   double* sc_out) {
  double sres[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sres[i] = i < cnt ? dot16<kPlaced>(x[i], y[i], qt) : 0.0;
  const double v = blocks_reduce<4>(sres, lane);
  if (lane < cnt) {
    sc_out[g0 + lane] = v;
    a.scores[(size_t)u * a.max_blocks + g0 + lane] = v;
  }
}

// Scores of every closed block of unit u by `nwarps` warps of one CTA, read
// straight from global memory: warp w takes the groups of 4 consecutive
// blocks starting at 4w, 4(w + nwarps), ...; two groups' loads are in flight
// (the first two issued before the queries are read) while a group is reduced.  The scores go to sc_out
// (shared memory) and to the caller's global buffer.  Same arithmetic as
// score_kernel.  With a.q_copy set, the unit's query rows are read once by
// the CTA (they may be in host memory), kept in q_stage (G * 16 uint4 of
// shared memory) and copied to a.q_copy; this takes a CTA-wide barrier, so
// every thread of the CTA must call.
__device__ __forceinline__ void score_unit_warps(const ScoreArgs& a, int u, int warp, int nwarps, int lane,
                                                 double* sc_out, uint4* q_stage = nullptr) {
  const int n = a.ds->n_closed;
  const int r = lane >> 3, c = lane & 7;
  const uint4* base = reinterpret_cast<const uint4*>(a.kbar) + (size_t)u * a.max_blocks * kBlockU4 + r * kRowU4;
  const int stride = nwarps * 4;
  uint4 xa[4], ya[4], xb[4], yb[4];
  int g = warp * 4;
  // the first two groups' keys and the queries travel together
  if (g < n) score_group_load(base, g, min(4, n - g), c, xa, ya);
  int g1 = g + stride;
  if (g1 < n) score_group_load(base, g1, min(4, n - g1), c, xb, yb);
  double qt[16];
  if (a.q_copy) {
    const size_t row0 = ((size_t)(u / a.Hkv) * a.Hq + (size_t)(u % a.Hkv) * a.G) * kRowU4;
    const uint4* src = reinterpret_cast<const uint4*>(a.q) + row0;
    uint4* dst = reinterpret_cast<uint4*>(a.q_copy) + row0;
    for (int i = warp * 32 + lane; i < a.G * kRowU4; i += nwarps * 32) {
      const uint4 v = src[i];
      q_stage[i] = v;
      dst[i] = v;
    }
    __syncthreads();
    group_query_sum(a, u / a.Hkv, u % a.Hkv, c, qt, q_stage);
  } else {
    group_query_sum(a, u / a.Hkv, u % a.Hkv, c, qt);
  }
  // two groups in flight: each finished group's buffer takes the group after next
  auto groups = [&](auto placed) {
    constexpr bool kPlaced = decltype(placed)::value;
    while (g < n) {
      score_group_finish<kPlaced>(a, u, g, min(4, n - g), lane, xa, ya, qt, sc_out);
      const int g2 = g1 + stride;
      if (g2 < n) score_group_load(base, g2, min(4, n - g2), c, xa, ya);
      if (g1 >= n) break;
      score_group_finish<kPlaced>(a, u, g1, min(4, n - g1), lane, xb, yb, qt, sc_out);
      const int g3 = g2 + stride;
      if (g3 < n) score_group_load(base, g3, min(4, n - g3), c, xb, yb);
      g = g2;
      g1 = g3;
    }
  };
  if (a.placed_widen && place_query_terms(qt)) {
    groups(std::true_type{});
  } else {
    groups(std::false_type{});
  }
}

}  // namespace nosa
