// decode.cu -- block-sparse GQA attention over the selected blocks, split-KV
// partials and their combine, plus the per-step state kernels (tail append,
// block close, step advance).
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), App. A:
// after the misses arrive, attention is computed with the GPU-resident KV
// blocks.  Each query head attends to the 64 tokens of every selected block of
// its KV head (plus the open tail block), softmax scaled by 1/sqrt(d).
//
// Kernel layout (one CTA = one unit x one split of its block list):
//  * K and V blocks (64 tokens x 128 dims bf16, 16 KiB each) are staged in
//    shared memory by 2-D TMA loads with the 128-byte swizzle, three blocks in
//    flight, completion tracked by mbarriers.
//  * Four warps each own 16 tokens of a block.  Scores S^T[token][head] come
//    from mma.m16n8k16 with the block as A (tokens x dims) and the query group
//    as B (dims x 8 heads; heads >= G are zero), so the 4-head group wastes half
//    of N rather than 3/4 of M.  P^T is moved into the B layout with movmatrix
//    and O^T[dim][head] += V^T P^T uses ldmatrix.trans on the V tile.
//  * Online softmax per warp in the exp2 domain; the four warps and then the
//    splits are merged by log-sum-exp weights.
#include <cfloat>

#include "nosa_internal.cuh"

namespace nosa {

constexpr int kStages = 3;
constexpr int kDecThreads = 128;
constexpr int kHalfBytes = kP * 64 * 2;  // one 64-row x 64-dim box = 8 KiB
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct DecSmemLayout {
  static constexpr int kTile = kBlockBytes;        // 16 KiB
  static constexpr int kStage = 2 * kTile;         // K + V
  static constexpr int kBars = kStages * kStage;   // barrier offset
  static constexpr int kBytes = kBars + 64;
};

int decode_smem_bytes() { return DecSmemLayout::kBytes + 1024; }

// Final merge of one unit: the partials of parts [0, part_base) already in
// global memory plus (optionally) this CTA's four warps' states in shared
// memory; writes out[b, g*G + h, :] as bf16.
__device__ void merge_and_store(const DecodeArgs& a, int u, int b, int g, const float* sO, const float* sM,
                                const float* sL) {
  const float* po = a.part_o + (size_t)u * a.nparts * a.G * kD;
  const float2* pml = a.part_ml + (size_t)u * a.nparts * a.G;
  for (int idx = threadIdx.x; idx < a.G * kD; idx += blockDim.x) {
    const int h = idx / kD, dd = idx % kD;
    float M = -INFINITY;
    for (int p = 0; p < a.part_base; ++p) M = fmaxf(M, pml[p * a.G + h].x);
    if (sM) {
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, sM[w * kMaxG + h]);
    }
    const float Mu = M == -INFINITY ? 0.f : M;
    float num = 0.f, den = 0.f;
    for (int p = 0; p < a.part_base; ++p) {
      const float2 ml = pml[p * a.G + h];
      if (ml.y <= 0.f) continue;
      const float f = exp2f(ml.x - Mu);
      num += f * po[((size_t)p * a.G + h) * kD + dd];
      den += f * ml.y;
    }
    if (sM) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float l = sL[w * kMaxG + h];
        if (l <= 0.f) continue;
        const float f = exp2f(sM[w * kMaxG + h] - Mu);
        num += f * sO[(w * kMaxG + h) * kD + dd];
        den += f * l;
      }
    }
    const float r = den > 0.f ? num / den : 0.f;
    a.out[((size_t)b * a.Hq + (size_t)g * a.G + h) * kD + dd] = (uint16_t)(pack_bf16x2(r, 0.f) & 0xFFFFu);
  }
}

__global__ void __launch_bounds__(kDecThreads, 2)
    decode_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_tk, const __grid_constant__ CUtensorMap map_tv,
                  DecodeArgs a) {
  const int u = blockIdx.y, s = blockIdx.x;
  const int b = u / a.Hkv, g = u % a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool tail = a.tail_split && s == a.splits;

  // ---- the item range of this split
  int lo = 0, hi = 0, len = kP;
  if (tail) {
    len = a.ds->tail_len_step;
    hi = len > 0 ? 1 : 0;
  } else {
    int base_lo, base_hi;
    if (a.resident) {
      base_lo = 0;
      base_hi = a.k;
    } else if (a.phase == 1) {
      base_lo = 0;
      base_hi = a.n_hit[u];
    } else {
      base_lo = a.n_hit[u];
      base_hi = a.n_items[u];
    }
    if (a.merge_out) {  // one CTA per unit takes every remaining item
      lo = base_lo;
      hi = base_hi;
    } else {
      lo = base_lo + s * a.bps;
      hi = min(base_lo + (s + 1) * a.bps, base_hi);
    }
  }
  const int n_it = hi > lo ? hi - lo : 0;
  const size_t part = (size_t)u * a.nparts + a.part_base + s;
  float* po = a.part_o + part * a.G * kD;
  float2* pml = a.part_ml + part * a.G;

  extern __shared__ unsigned char dsm_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                                       ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + DecSmemLayout::kBars);
  if (n_it == 0) {
    if (a.merge_out) {
      merge_and_store(a, u, b, g, nullptr, nullptr, nullptr);
    } else if (threadIdx.x < a.G) {
      pml[threadIdx.x] = make_float2(-INFINITY, 0.f);
    }
    return;
  }

  // ---- producer: thread 0 issues one block's K and V (4 boxes, 32 KiB)
  auto issue = [&](int it, int st) {
    const CUtensorMap* mk = &map_k;
    const CUtensorMap* mv = &map_v;
    int row;
    if (tail) {
      mk = &map_tk;
      mv = &map_tv;
      row = u * kP;
    } else if (a.resident) {
      int blk = a.sel[(size_t)u * a.k + lo + it];
      if (blk < 0 || blk >= a.max_blocks) {
        atomicOr(&a.ds->error_bits, ERR_RANGE);
        blk = 0;
      }
      row = (u * a.max_blocks + blk) * kP;
    } else {
      int slot = a.items[(size_t)u * a.k + lo + it];
      if (slot < 0 || slot >= a.C) {
        atomicOr(&a.ds->error_bits, ERR_RANGE);
        slot = 0;
      }
      row = (u * a.C + slot) * kP;
    }
    unsigned char* kt = sm + st * DecSmemLayout::kStage;
    unsigned char* vt = kt + DecSmemLayout::kTile;
    mbar_arrive_expect_tx(&bars[st], 2 * kBlockBytes);
    tma_load_2d(kt, mk, &bars[st], 0, row);
    tma_load_2d(kt + kHalfBytes, mk, &bars[st], 64, row);
    tma_load_2d(vt, mv, &bars[st], 0, row);
    tma_load_2d(vt + kHalfBytes, mv, &bars[st], 64, row);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages && i < n_it; ++i) issue(i, i);
  }

  // ---- query group as the mma B operand: lane holds head lane/4,
  // dims 16 ks + 2 (lane%4) + {0,1} and + 8
  uint32_t qf[8][2];
  {
    const int hb = lane >> 2;
    const uint32_t* qrow =
        reinterpret_cast<const uint32_t*>(a.q + ((size_t)b * a.Hq + (size_t)g * a.G + (hb < a.G ? hb : 0)) * kD);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qf[ks][0] = hb < a.G ? qrow[ks * 8 + (lane & 3)] : 0u;
      qf[ks][1] = hb < a.G ? qrow[ks * 8 + 4 + (lane & 3)] : 0u;
    }
  }

  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sc = 0.088388347648318440f * 1.4426950408889634f;  // log2(e) / sqrt(128)

  const int tok_a = warp * 16 + (lane & 15);                          // ldmatrix row, K
  const int tok_v = warp * 16 + (lane & 7) + ((lane >> 4) << 3);     // ldmatrix row, V (trans)
  const int t0 = warp * 16 + (lane >> 2), t1 = t0 + 8;                // accumulator rows

  bool timed_out = false;
  int consumed = 0;
  for (int it = 0; it < n_it; ++it) {
    const int st = it % kStages;
    const bool ok = mbar_wait_bounded(&bars[st], (uint32_t)((it / kStages) & 1), kWaitLimitNs);
    if (__syncthreads_or(!ok)) {  // every thread takes the same exit
      timed_out = true;
      break;
    }
    consumed = it + 1;
    const uint32_t kb = smem_u32(sm + st * DecSmemLayout::kStage);
    const uint32_t vb = kb + DecSmemLayout::kTile;

    // S^T (16 tokens x 8 heads) for this warp's tokens
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int chunk = 2 * ks + (lane >> 4);
      const uint32_t addr = kb + (chunk >> 3) * kHalfBytes + tok_a * 128 + (((chunk & 7) ^ (tok_a & 7)) << 4);
      uint32_t a0, a1, a2, a3;
      ldsm_x4(addr, a0, a1, a2, a3);
      mma_bf16_16816(c, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
    }
    const float s0 = t0 < len ? c[0] * sc : -INFINITY;
    const float s1 = t0 < len ? c[1] * sc : -INFINITY;
    const float s2 = t1 < len ? c[2] * sc : -INFINITY;
    const float s3 = t1 < len ? c[3] * sc : -INFINITY;
    float bm0 = fmaxf(s0, s2), bm1 = fmaxf(s1, s3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
      bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
    }
    const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
    const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = exp2f(m0 - mu0), al1 = exp2f(m1 - mu1);
    const float p0 = exp2f(s0 - mu0), p1 = exp2f(s1 - mu1);
    const float p2 = exp2f(s2 - mu0), p3 = exp2f(s3 - mu1);
    l0 = l0 * al0 + p0 + p2;
    l1 = l1 * al1 + p1 + p3;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      o[mt][0] *= al0; o[mt][1] *= al1; o[mt][2] *= al0; o[mt][3] *= al1;
    }
    const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int chunk = 2 * mt + ((lane >> 3) & 1);
      const uint32_t addr = vb + (chunk >> 3) * kHalfBytes + tok_v * 128 + (((chunk & 7) ^ (tok_v & 7)) << 4);
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(addr, a0, a1, a2, a3);
      mma_bf16_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
    }
    __syncthreads();
    if (threadIdx.x == 0 && it + kStages < n_it) issue(it + kStages, st);
  }

  if (timed_out) {
    // record, then give the loads already issued a bounded chance to land
    if (threadIdx.x == 0) {
      atomicOr(&a.ds->error_bits, ERR_TIMEOUT);
      const int issued = min(n_it, consumed + kStages);
      for (int it = consumed; it < issued; ++it)
        (void)mbar_wait_bounded(&bars[it % kStages], (uint32_t)((it / kStages) & 1), kWaitLimitNs);
    }
    __syncthreads();
    if (!a.merge_out && threadIdx.x < a.G) pml[threadIdx.x] = make_float2(-INFINITY, 0.f);
    return;
  }

  // ---- merge the four warps (stage buffers are free now)
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  float* sO = reinterpret_cast<float*>(sm);                 // [4 warps][8 heads][128]
  float* sM = sO + 4 * kMaxG * kD;                           // [4][8]
  float* sL = sM + 4 * kMaxG;                                // [4][8]
  const int h0 = (lane & 3) * 2, h1 = h0 + 1;
  if (lane < 4) {
    sM[warp * kMaxG + h0] = m0; sM[warp * kMaxG + h1] = m1;
    sL[warp * kMaxG + h0] = l0; sL[warp * kMaxG + h1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d0 = mt * 16 + (lane >> 2);
    float* w = sO + warp * kMaxG * kD;
    w[h0 * kD + d0] = o[mt][0];
    w[h1 * kD + d0] = o[mt][1];
    w[h0 * kD + d0 + 8] = o[mt][2];
    w[h1 * kD + d0 + 8] = o[mt][3];
  }
  __syncthreads();
  if (a.merge_out) {
    merge_and_store(a, u, b, g, sO, sM, sL);
    return;
  }
  for (int idx = threadIdx.x; idx < a.G * kD; idx += kDecThreads) {
    const int h = idx / kD, dd = idx % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sM[w * kMaxG + h]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float f = exp2f(sM[w * kMaxG + h] - Mu);
      acc += f * sO[(w * kMaxG + h) * kD + dd];
      L += f * sL[w * kMaxG + h];
    }
    po[h * kD + dd] = acc;
    if (dd == 0) pml[h] = make_float2(M, L);
  }
}

// Called once per context creation (on its device), outside any stream capture.
cudaError_t configure_decode() {
  return cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, decode_smem_bytes());
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t st) {
  const int smem = decode_smem_bytes();
  dim3 grid(a.splits + (a.tail_split ? 1 : 0), a.U);
  decode_kernel<<<grid, kDecThreads, smem, st>>>(m.k, m.v, m.tk, m.tv, a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- combine
// out[b, g*G + h, :] = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p
__global__ void __launch_bounds__(128) combine_kernel(CombineArgs a) {
  const int u = blockIdx.x;
  const int b = u / a.Hkv, g = u % a.Hkv;
  const float* po = a.part_o + (size_t)u * a.nparts * a.G * kD;
  const float2* pml = a.part_ml + (size_t)u * a.nparts * a.G;
  for (int idx = threadIdx.x; idx < a.G * kD; idx += blockDim.x) {
    const int h = idx / kD, dd = idx % kD;
    float M = -INFINITY;
    for (int p = 0; p < a.nparts; ++p) M = fmaxf(M, pml[p * a.G + h].x);
    const float Mu = M == -INFINITY ? 0.f : M;
    float num = 0.f, den = 0.f;
    for (int p = 0; p < a.nparts; ++p) {
      const float2 ml = pml[p * a.G + h];
      if (ml.y <= 0.f) continue;
      const float f = exp2f(ml.x - Mu);
      num += f * po[((size_t)p * a.G + h) * kD + dd];
      den += f * ml.y;
    }
    const float r = den > 0.f ? num / den : 0.f;
    const uint32_t bits = pack_bf16x2(r, 0.f) & 0xFFFFu;
    a.out[((size_t)b * a.Hq + (size_t)g * a.G + h) * kD + dd] = (uint16_t)bits;
  }
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
  combine_kernel<<<a.U, 128, 0, st>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- tail append
// One token per unit goes to row tail_len of the open tail block.  The new
// length is published in tail_len_step by one thread; every thread of this
// launch reads only tail_len.
__global__ void __launch_bounds__(32) append_kernel(AppendArgs a) {
  const int u = blockIdx.x;
  const int tl = a.ds->tail_len;
  const int n = a.ds->n_closed;
  const bool ok = tl < kP && (n * kP + tl + 1) <= a.max_blocks * kP;
  if (u == 0 && threadIdx.x == 0) {
    if (ok) a.ds->tail_len_step = tl + 1;
    else atomicOr(&a.ds->error_bits, ERR_CAPACITY);
  }
  if (!ok) return;
  const uint4* sk = reinterpret_cast<const uint4*>(a.k_new) + (size_t)u * kRowU4;
  const uint4* sv = reinterpret_cast<const uint4*>(a.v_new) + (size_t)u * kRowU4;
  uint4* dk = reinterpret_cast<uint4*>(a.tail_k) + ((size_t)u * kP + tl) * kRowU4;
  uint4* dv = reinterpret_cast<uint4*>(a.tail_v) + ((size_t)u * kP + tl) * kRowU4;
  if (threadIdx.x < kRowU4) dk[threadIdx.x] = sk[threadIdx.x];
  else if (threadIdx.x < 2 * kRowU4) dv[threadIdx.x - kRowU4] = sv[threadIdx.x - kRowU4];
  if (threadIdx.x == 0 && a.a_close) a.a_pending[u] = a.a_close[u];
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t st) {
  append_kernel<<<a.U, 32, 0, st>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- block close
// When the tail holds P tokens at the end of a step, it becomes closed block
// n: its pooled keys are built (same rule as at attach), its agnostic score is
// registered, and K/V are written through to the attached KV store.
__global__ void __launch_bounds__(256) close_kernel(CloseArgs a) {
  const int u = blockIdx.x;
  if (a.ds->tail_len_step != kP) return;
  const int n = a.ds->n_closed;
  if (n >= a.max_blocks) {
    if (threadIdx.x == 0) atomicOr(&a.ds->error_bits, ERR_CAPACITY);
    return;
  }
  const uint4* tk = reinterpret_cast<const uint4*>(a.tail_k) + (size_t)u * kP * kRowU4;
  const uint4* tv = reinterpret_cast<const uint4*>(a.tail_v) + (size_t)u * kP * kRowU4;
  if (threadIdx.x < kR * 16) {
    const int sb = threadIdx.x >> 4, c = threadIdx.x & 15;
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    for (int j = 0; j < kQ; ++j) {
      const uint4 w = tk[(size_t)(sb * kQ + j) * kRowU4 + c];
      acc[0] += bf16_lo_to_f64(w.x); acc[1] += bf16_hi_to_f64(w.x);
      acc[2] += bf16_lo_to_f64(w.y); acc[3] += bf16_hi_to_f64(w.y);
      acc[4] += bf16_lo_to_f64(w.z); acc[5] += bf16_hi_to_f64(w.z);
      acc[6] += bf16_lo_to_f64(w.w); acc[7] += bf16_hi_to_f64(w.w);
    }
    uint32_t ob[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) ob[i] = f64_to_bf16_bits(acc[i] * (1.0 / kQ));
    uint4* kb = reinterpret_cast<uint4*>(a.kbar) + (((size_t)u * a.max_blocks + n) * kR + sb) * kRowU4 + c;
    *kb = make_uint4(ob[0] | (ob[1] << 16), ob[2] | (ob[3] << 16), ob[4] | (ob[5] << 16),
                     ob[6] | (ob[7] << 16));
  }
  uint4* dk = reinterpret_cast<uint4*>(a.kv_k) + ((size_t)u * a.max_blocks + n) * kP * kRowU4;
  uint4* dv = reinterpret_cast<uint4*>(a.kv_v) + ((size_t)u * a.max_blocks + n) * kP * kRowU4;
  for (int i = threadIdx.x; i < kP * kRowU4; i += blockDim.x) {
    dk[i] = tk[i];
    dv[i] = tv[i];
  }
  if (threadIdx.x == 0) a.agnostic[(size_t)u * a.max_blocks + n] = a.a_pending[u];
}

cudaError_t launch_close(const CloseArgs& a, cudaStream_t st) {
  close_kernel<<<a.U, 256, 0, st>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- step state
__global__ void advance_kernel(DevState* ds, DevStats* st) {
  ds->n_last_select = ds->n_closed;
  const int tl = ds->tail_len_step;
  if (tl >= kP) {
    ds->n_closed += 1;
    ds->tail_len = 0;
  } else {
    ds->tail_len = tl;
  }
  ds->tail_len_step = ds->tail_len;
  ds->step += 1;
  st->steps += 1;
}

cudaError_t launch_advance(DevState* ds, DevStats* st, cudaStream_t s) {
  advance_kernel<<<1, 1, 0, s>>>(ds, st);
  return cudaGetLastError();
}

__global__ void init_state_kernel(DevState* ds, int n_closed, int tail_len, int step, int n_last_select) {
  ds->step = step;
  ds->n_closed = n_closed;
  ds->n_last_select = n_last_select;
  ds->tail_len = tail_len;
  ds->tail_len_step = tail_len;
  ds->gather_count = 0;
  ds->error_bits = 0u;
  ds->pad = 0;
}

cudaError_t launch_init_state(DevState* ds, int n_closed, int tail_len, int step, int n_last_select,
                              cudaStream_t s) {
  init_state_kernel<<<1, 1, 0, s>>>(ds, n_closed, tail_len, step, n_last_select);
  return cudaGetLastError();
}

__global__ void reset_stats_kernel(DevStats* st) {
  st->steps = st->selected = st->hits = st->misses = st->fetched_bytes = 0ull;
  st->overlap_sum = st->overlap_terms = 0ull;
  st->min_overlap = 0x7fffffff;
  st->max_fetch = 0;
}

cudaError_t launch_reset_stats(DevStats* st, cudaStream_t s) {
  reset_stats_kernel<<<1, 1, 0, s>>>(st);
  return cudaGetLastError();
}

// Bounded wait on a flag that another agent (host or kernel) sets.
__global__ void wait_flag_kernel(const volatile int* flag, DevState* ds, long long timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; it < (1u << 30); ++it) {
    if (*flag != 0) return;
    if (global_timer_ns() - t0 > (uint64_t)timeout_ns) break;
    __nanosleep(1000);
  }
  atomicOr(&ds->error_bits, ERR_TIMEOUT);
}

cudaError_t launch_wait_flag(const volatile int* flag, DevState* ds, long long timeout_ns, cudaStream_t s) {
  wait_flag_kernel<<<1, 1, 0, s>>>(flag, ds, timeout_ns);
  return cudaGetLastError();
}

}  // namespace nosa
