// state.cu -- per-step state kernels: tail append, block close, step
// advance, state initialisation, statistics reset and the bounded flag wait.
//
// NOSA: Native and Offloadable Sparse Attention (paperlayer summary), App. A
// (reading for growing sequences): a token appended at step t goes into the
// open tail block; a full tail becomes a closed block at the end of the step,
// with its pooled keys built as at attach time and its K/V written through to
// the attached KV store.
#include "nosa_internal.cuh"

namespace nosa {

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
// n: its pooled keys are built (same rule as at attach) and its agnostic score
// is registered.  Its K/V go to the attached KV store directly when that store
// is in HBM.  When the store is in host memory they go to a staging buffer in
// HBM instead, and write_through_kernel moves them to the host during the next
// step, off the critical path; until the next close the gather reads block n
// from the staging copy.
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
  const bool staged = a.stage_k != nullptr;
  const size_t dst = staged ? (size_t)u * kP * kRowU4 : ((size_t)u * a.max_blocks + n) * kP * kRowU4;
  uint4* dk = reinterpret_cast<uint4*>(staged ? a.stage_k : a.kv_k) + dst;
  uint4* dv = reinterpret_cast<uint4*>(staged ? a.stage_v : a.kv_v) + dst;
  for (int i = threadIdx.x; i < kP * kRowU4; i += blockDim.x) {
    dk[i] = tk[i];
    dv[i] = tv[i];
  }
  if (threadIdx.x == 0) a.agnostic[(size_t)u * a.max_blocks + n] = a.a_pending[u];
  if (staged && u == 0 && threadIdx.x == 0) {
    a.ds->staged_block = n;
    a.ds->wt_block = n;
  }
}

cudaError_t launch_close(const CloseArgs& a, cudaStream_t st) {
  close_kernel<<<a.U, 256, 0, st>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- write-through
// Copies the staged block of every unit into the host KV store with
// zero-copy stores (device-to-host over PCIe, the direction the miss gather
// does not use).  The launch that finds a block pending clears the flag from
// its last CTA; a launch with nothing pending returns at once.
__global__ void __launch_bounds__(256) write_through_kernel(WriteThroughArgs a) {
  const int n = a.ds->wt_block;
  if (n < 0) return;
  if (n >= a.max_blocks) {
    if (threadIdx.x == 0) atomicOr(&a.ds->error_bits, ERR_RANGE);
    return;
  }
  for (int u = blockIdx.x; u < a.U; u += gridDim.x) {
    const uint4* sk = reinterpret_cast<const uint4*>(a.stage_k) + (size_t)u * kP * kRowU4;
    const uint4* sv = reinterpret_cast<const uint4*>(a.stage_v) + (size_t)u * kP * kRowU4;
    uint4* dk = reinterpret_cast<uint4*>(a.kv_k) + ((size_t)u * a.max_blocks + n) * kP * kRowU4;
    uint4* dv = reinterpret_cast<uint4*>(a.kv_v) + ((size_t)u * a.max_blocks + n) * kP * kRowU4;
    uint4 rk[kP * kRowU4 / 256], rv[kP * kRowU4 / 256];
#pragma unroll
    for (int i = 0; i < kP * kRowU4 / 256; ++i) {
      rk[i] = sk[threadIdx.x + i * 256];
      rv[i] = sv[threadIdx.x + i * 256];
    }
#pragma unroll
    for (int i = 0; i < kP * kRowU4 / 256; ++i) {
      dk[threadIdx.x + i * 256] = rk[i];
      dv[threadIdx.x + i * 256] = rv[i];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence_system();
    if (atomicAdd(&a.ds->wt_done, 1) == (int)gridDim.x - 1) {
      a.ds->wt_block = -1;
      a.ds->wt_done = 0;
    }
  }
}

cudaError_t launch_write_through(const WriteThroughArgs& a, int grid, cudaStream_t st) {
  int least = 0, greatest = 0;
  cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributePriority;
  attr[0].val.priority = least;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, write_through_kernel, a);
}

// ---------------------------------------------------------------- step state
__global__ void advance_kernel(DevState* ds, DevStats* st) { advance_step(ds, st); }

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
  ds->staged_block = -1;
  ds->wt_block = -1;
  ds->wt_done = 0;
  ds->gather_next = 0;
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
