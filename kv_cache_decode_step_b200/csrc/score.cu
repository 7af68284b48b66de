// score.cu -- pooled keys and two-stage block scoring.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), §3.1:
// blocks are scored in two stages, mean pooling over sub-blocks and then max
// pooling over the sub-blocks of a block.  Here a sub-block is 16 tokens and a
// block 64 (4 sub-blocks); the sub-block score of KV head g sums the raw dot
// products of its G query heads with the pooled key.
#include "score_dev.cuh"

namespace nosa {

// ---------------------------------------------------------------- pooling
// Block of 256 threads = 16 sub-blocks x 16 lanes; a lane owns 8 dims (16 B).
// The 16 keys of a sub-block are summed exactly in fp64 (bf16 inputs), divided
// by 16 (exact) and rounded once to bf16.
__global__ void __launch_bounds__(256) pool_kernel(const uint4* __restrict__ src, size_t src_unit_tokens,
                                                   int s_begin, int s_end, uint4* __restrict__ kbar,
                                                   int kbar_unit_rows) {
  const int u = blockIdx.y;
  const int s = s_begin + blockIdx.x * 16 + (threadIdx.x >> 4);
  if (s >= s_end) return;
  const int c = threadIdx.x & 15;
  const uint4* p = src + ((size_t)u * src_unit_tokens + (size_t)s * kQ) * kRowU4 + c;
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  uint4 w[kQ];
#pragma unroll
  for (int j = 0; j < kQ; ++j) w[j] = p[(size_t)j * kRowU4];
#pragma unroll
  for (int j = 0; j < kQ; ++j) {
    acc[0] += bf16_lo_to_f64(w[j].x); acc[1] += bf16_hi_to_f64(w[j].x);
    acc[2] += bf16_lo_to_f64(w[j].y); acc[3] += bf16_hi_to_f64(w[j].y);
    acc[4] += bf16_lo_to_f64(w[j].z); acc[5] += bf16_hi_to_f64(w[j].z);
    acc[6] += bf16_lo_to_f64(w[j].w); acc[7] += bf16_hi_to_f64(w[j].w);
  }
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = f64_to_bf16_bits(acc[i] * (1.0 / kQ));
  uint4 r;
  r.x = o[0] | (o[1] << 16);
  r.y = o[2] | (o[3] << 16);
  r.z = o[4] | (o[5] << 16);
  r.w = o[6] | (o[7] << 16);
  kbar[((size_t)u * kbar_unit_rows + s) * kRowU4 + c] = r;
}

cudaError_t launch_pool(const uint16_t* src, size_t src_unit_tokens, int U, int s_begin, int s_end,
                        uint16_t* kbar, int kbar_unit_rows, cudaStream_t st) {
  if (s_end <= s_begin || U <= 0) return cudaSuccess;
  dim3 grid((s_end - s_begin + 15) / 16, U);
  pool_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(src), src_unit_tokens, s_begin, s_end,
                                    reinterpret_cast<uint4*>(kbar), kbar_unit_rows);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- scoring
// One CTA = one unit x 32 blocks (32 KiB of pooled keys), four warps of 8
// blocks.  Thread 0 starts four bulk copies of the CTA's pooled keys into
// shared memory at once (seven CTAs per SM: the whole batch is in flight in
// one wave) and each warp waits only for its own 8 blocks.  Within a block,
// lanes 8r..8r+7 hold sub-block r and lane 8r+c owns dims [8c, 8c+8) and
// [64+8c, 64+8c+8), so every quarter-warp reads 128 contiguous bytes.
// The group's queries are summed first (fp64, exact for bf16 inputs), so each
// sub-block score is one 128-term fp64 dot product whose products are exact;
// only the summation order differs from the definition.
constexpr int kScoreCtaBlocks = 32;
constexpr int kScoreWarps = 4;
constexpr int kScoreWarpBlocks = kScoreCtaBlocks / kScoreWarps;
constexpr uint64_t kScoreWaitNs = 1000000000ull;

__global__ void __launch_bounds__(kScoreWarps * 32) score_kernel(ScoreArgs a) {
  __shared__ __align__(128) uint4 skb[kScoreCtaBlocks * kBlockU4];  // 32 KiB
  __shared__ __align__(8) uint64_t bars[kScoreWarps];
  grid_dep_launch();  // a selection launched as a dependent may be placed; it waits for the scores
  const int u = blockIdx.y;
  const int n = a.ds->n_closed;
  const int j0 = blockIdx.x * kScoreCtaBlocks;
  if (j0 >= n) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = min(kScoreCtaBlocks, n - j0);
  const uint4* src = reinterpret_cast<const uint4*>(a.kbar) + ((size_t)u * a.max_blocks + j0) * kBlockU4;
  if (threadIdx.x == 0) {
    for (int w = 0; w < kScoreWarps; ++w) mbar_init(&bars[w], 1);
    fence_mbar_init();
    for (int w = 0; w < kScoreWarps; ++w) {
      const int cnt = min(kScoreWarpBlocks, nb - w * kScoreWarpBlocks);
      if (cnt <= 0) break;
      const uint32_t bytes = (uint32_t)cnt * kBlockU4 * 16;
      mbar_arrive_expect_tx(&bars[w], bytes);
      bulk_load(skb + w * kScoreWarpBlocks * kBlockU4, src + (size_t)w * kScoreWarpBlocks * kBlockU4, bytes,
                &bars[w]);
    }
  }
  __syncthreads();

  const int r = lane >> 3, c = lane & 7;
  const int b = u / a.Hkv, g = u % a.Hkv;
  double qt[16];
  group_query_sum(a, b, g, c, qt);

  const int jw = warp * kScoreWarpBlocks;
  const int cnt = min(kScoreWarpBlocks, nb - jw);
  bool timed_out = false;
  if (cnt > 0) {
    if (!mbar_wait_bounded(&bars[warp], 0u, kScoreWaitNs)) {
      timed_out = true;
    } else {
      double sres[kScoreWarpBlocks];
      auto dots = [&](auto placed) {
        constexpr bool kPlaced = decltype(placed)::value;
#pragma unroll
        for (int i = 0; i < kScoreWarpBlocks; ++i) {
          if (i < cnt) {
            const uint4* row = skb + (jw + i) * kBlockU4 + r * kRowU4;
            sres[i] = dot16<kPlaced>(row[c], row[8 + c], qt);
          } else {
            sres[i] = 0.0;
          }
        }
      };
      if (a.placed_widen && place_query_terms(qt)) {
        dots(std::true_type{});
      } else {
        dots(std::false_type{});
      }
      const double v = blocks_reduce<kScoreWarpBlocks>(sres, lane);
      if (lane < cnt) a.scores[(size_t)u * a.max_blocks + j0 + jw + lane] = v;
    }
  }
  // never leave a bulk copy in flight behind an exiting CTA
  if (__syncthreads_or(timed_out) && threadIdx.x == 0) {
    atomicOr(&a.ds->error_bits, ERR_TIMEOUT);
    for (int w = 0; w < kScoreWarps; ++w)
      if (w * kScoreWarpBlocks < nb) (void)mbar_wait_bounded(&bars[w], 0u, kScoreWaitNs);
  }
}

cudaError_t launch_score(const ScoreArgs& a, cudaStream_t st) {
  dim3 grid((a.max_blocks + kScoreCtaBlocks - 1) / kScoreCtaBlocks, a.U);
  score_kernel<<<grid, kScoreWarps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nosa
