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

#include "nosa_internal.cuh"

namespace nosa {

constexpr int kBlockU4 = kR * kRowU4;  // 16-byte words of pooled keys per block (64)

__device__ __forceinline__ double dot16(const uint4& a, const uint4& b, const double* qt) {
  double s = 0.0;
  s = fma(qt[0], bf16_lo_to_f64(a.x), s);  s = fma(qt[1], bf16_hi_to_f64(a.x), s);
  s = fma(qt[2], bf16_lo_to_f64(a.y), s);  s = fma(qt[3], bf16_hi_to_f64(a.y), s);
  s = fma(qt[4], bf16_lo_to_f64(a.z), s);  s = fma(qt[5], bf16_hi_to_f64(a.z), s);
  s = fma(qt[6], bf16_lo_to_f64(a.w), s);  s = fma(qt[7], bf16_hi_to_f64(a.w), s);
  s = fma(qt[8], bf16_lo_to_f64(b.x), s);  s = fma(qt[9], bf16_hi_to_f64(b.x), s);
  s = fma(qt[10], bf16_lo_to_f64(b.y), s); s = fma(qt[11], bf16_hi_to_f64(b.y), s);
  s = fma(qt[12], bf16_lo_to_f64(b.z), s); s = fma(qt[13], bf16_hi_to_f64(b.z), s);
  s = fma(qt[14], bf16_lo_to_f64(b.w), s); s = fma(qt[15], bf16_hi_to_f64(b.w), s);
  return s;
}

__device__ __forceinline__ double block_reduce(double s) {
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  s += __shfl_xor_sync(0xffffffffu, s, 4);
  double o = __shfl_xor_sync(0xffffffffu, s, 8);
  s = o > s ? o : s;
  o = __shfl_xor_sync(0xffffffffu, s, 16);
  return o > s ? o : s;
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

__device__ __forceinline__ void score_group_finish(const ScoreArgs& a, int u, int g0, int cnt, int lane,
                                                   const uint4 (&x)[4], const uint4 (&y)[4], const double (&qt)[16],
                                                   double* sc_out) {
  double sres[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sres[i] = i < cnt ? dot16(x[i], y[i], qt) : 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) sres[i] = block_reduce(sres[i]);
  if (lane < cnt) {
    double v = sres[0];
#pragma unroll
    for (int i = 1; i < 4; ++i)
      if (lane == i) v = sres[i];
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
  while (g < n) {
    score_group_finish(a, u, g, min(4, n - g), lane, xa, ya, qt, sc_out);
    const int g2 = g1 + stride;
    if (g2 < n) score_group_load(base, g2, min(4, n - g2), c, xa, ya);
    if (g1 >= n) break;
    score_group_finish(a, u, g1, min(4, n - g1), lane, xb, yb, qt, sc_out);
    const int g3 = g2 + stride;
    if (g3 < n) score_group_load(base, g3, min(4, n - g3), c, xb, yb);
    g = g2;
    g1 = g3;
  }
}

}  // namespace nosa
