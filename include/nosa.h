/*
 * nosa.h -- C ABI of libnosa.so: the NOSA decode step on one B200 (sm_100a).
 *
 * NOSA (NOSA: Native and Offloadable Sparse Attention, paperlayer summary,
 * App. A) decodes each step as: select blocks -> move the cache-missed KV
 * blocks CPU -> GPU -> attend with the GPU-resident blocks.  This library
 * splits that step into four calls, made in this order once per step:
 *
 *   nosa_score_blocks   block scores from pooled keys        (§3.1)
 *   nosa_select         eviction-bounded query-agnostic set + capped
 *                       query-aware top-k, overlap >= m       (§3.1, App. E)
 *   nosa_fetch_missing  set difference against the GPU block cache: which
 *                       blocks miss and which slots they take (§4); it moves
 *                       no bytes
 *   nosa_sparse_decode  the zero-copy gather of the misses over PCIe (§4),
 *                       fused with the GQA attention over the selected
 *                       blocks (App. A)
 *
 * plus nosa_append_token first when the sequence grows during decoding.
 * nosa_score_select_fetch makes the first three calls in one (one kernel up
 * to 512 blocks per unit), and nosa_decode_step the whole step, with queries
 * and outputs in device or pinned host memory.
 *
 * Terms.  A unit is one (sequence b, KV head g), numbered u = b*n_kv_heads + g.
 * G = n_q_heads / n_kv_heads query heads share a KV head; query head h uses KV
 * head h / G.  A block is P = 64 tokens, a sub-block Q = 16 tokens, R = P/Q = 4
 * sub-blocks per block, head_dim d = 128.  n is the number of closed (full)
 * blocks of every unit; a partially filled last block (the tail) is attended
 * but never scored, selected or fetched.  k = k_query + k_agnostic.
 *
 * Conventions (every entry point):
 *  - Returns a nosa_status and never aborts, throws or exits.  On failure,
 *    nosa_last_error() gives a message for the calling thread.
 *  - "device" buffers are CUDA device memory of the context's device; "host"
 *    buffers are ordinary host memory; "pinned host" buffers are page-locked
 *    (cudaHostAlloc / cudaHostRegister) and therefore device-addressable.
 *  - Every buffer is owned by the caller, who keeps it alive and unmodified
 *    until the work queued on the stream that reads it has finished.
 *  - Calls are asynchronous on the given stream unless marked "synchronous".
 *    A CUDA error raised by earlier work may surface in a later call as
 *    NOSA_ERR_CUDA.  The step calls enqueue work only; they are safe to
 *    capture in a CUDA graph, and every per-step quantity (step counter, block
 *    count, tail length) lives in device memory so that replays advance it.
 *  - Out-of-order step calls return NOSA_ERR_ORDER and enqueue nothing.
 *  - A context is not thread-safe; use one context per thread or serialise.
 *  - Device-side waits are bounded (about 1 s).  A wait that runs out sets an
 *    error bit that nosa_check_errors() reports as NOSA_ERR_TIMEOUT.
 */
#ifndef NOSA_H
#define NOSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NOSA_API __attribute__((visibility("default")))
#else
#define NOSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA header.
 * NULL means the legacy default stream. */
typedef struct CUstream_st* nosa_stream_t;

typedef enum {
  NOSA_OK = 0,
  NOSA_ERR_INVALID = -1,        /* bad argument, config or pointer kind */
  NOSA_ERR_CUDA = -2,           /* a CUDA runtime/driver call failed */
  NOSA_ERR_NOMEM = -3,          /* device allocation failed */
  NOSA_ERR_ORDER = -4,          /* step calls out of order */
  NOSA_ERR_TIMEOUT = -5,        /* a bounded device-side wait ran out */
  NOSA_ERR_UNIMPLEMENTED = -6   /* configuration outside what v1 supports */
} nosa_status;

typedef struct nosa_ctx nosa_ctx;

/* Shape and budget of a decode batch.  v1 supports head_dim = 128, block = 64,
 * sub_block = 16 and 1 <= G <= 8 (otherwise NOSA_ERR_UNIMPLEMENTED). */
typedef struct {
  int batch;          /* B >= 1 sequences */
  int n_q_heads;      /* H_q, a multiple of n_kv_heads */
  int n_kv_heads;     /* H_kv >= 1 */
  int head_dim;       /* d, must be 128 */
  int block;          /* P, must be 64 */
  int sub_block;      /* Q, must be 16 */
  int k_query;        /* k_q >= 0 query-aware blocks per unit and step */
  int k_agnostic;     /* k_e >= 0 query-agnostic blocks per unit and step */
  int min_overlap;    /* m = ceil(gamma0 * k), 0 <= m <= k: at least m blocks
                         of S(t) were also in S(t-1) (NOSA summary §3.1) */
  int max_blocks;     /* block capacity per unit (prompt + growth), >= k, <= 8192 */
  int cache_slots;    /* 0: KV resident in HBM; else GPU cache blocks per unit,
                         k <= cache_slots <= 1024, KV in pinned host memory */
  int sink_blocks;    /* forced: the first sink_blocks closed blocks (attention sink) */
  int window_blocks;  /* forced: the last window_blocks closed blocks (sliding window);
                         sink + window <= k_agnostic: forced blocks count inside the
                         query-agnostic budget (NOSA summary App. B.2.2) */
} nosa_config;

/* Running totals since the last attach or nosa_reset_stats. */
typedef struct {
  int64_t steps;           /* decode steps completed (nosa_sparse_decode calls) */
  int64_t selected;        /* sum over units and steps of |S(t)| */
  int64_t hits;            /* selected blocks already in the GPU cache */
  int64_t misses;          /* selected blocks fetched over PCIe */
  int64_t fetched_bytes;   /* K+V bytes moved host -> device by the gather */
  int64_t overlap_sum;     /* sum over units, steps t >= 1 of |S(t) ∩ S(t-1)| */
  int64_t overlap_terms;   /* number of (unit, step >= 1) terms in overlap_sum */
  int32_t min_overlap;     /* min over units, steps t >= 1 of |S(t) ∩ S(t-1)|
                              (INT32_MAX before step 1) */
  int32_t max_fetch;       /* max over units, steps t >= 1 of blocks fetched */
  uint32_t error_bits;     /* device error bits (see nosa_check_errors) */
  int32_t n_closed;        /* closed blocks per unit now */
  int32_t tail_len;        /* tokens in the open tail block now */
  int32_t reserved;
} nosa_stats;

/* Validate cfg and allocate the context's device state on the current device:
 * pooled keys bf16 [U, max_blocks*R, d], agnostic scores fp32 [U, max_blocks],
 * selection state, the GPU block cache bf16 [U, cache_slots, P, d] x 2 (K, V)
 * with its tables, the open tail block bf16 [U, P, d] x 2 and attention
 * partials.  Synchronous.  *out is set only on NOSA_OK.
 *
 * Launch shapes are sized from the device's SM count and may be overridden by
 * environment variables read here, once per context.  None changes a score,
 * selection, fetch list or cache map.  These change no bit of the output
 * either: NOSA_GATHER_CTAS (gather CTAs), NOSA_ATTN_PRODUCER=0 (hits pass
 * without its producer warp), NOSA_KV_EVICT_FIRST=0 (hits-pass K/V loads
 * without the L2 evict-first policy), NOSA_PDL=0 (gather not launched as a
 * programmatic dependent of the plan), NOSA_PLACED_WIDEN=0 (scoring widens
 * every key by conversion) and NOSA_WARM_BLOCKS (0..64, default 12: KV in HBM,
 * blocks per hits-pass CTA prefetched into L2 during the selection).
 * NOSA_ATTN_CTAS, NOSA_ATTN_STAGES (2 or 3) and NOSA_ATTN_GAP (0..64 empty
 * positions per unit) change the hits pass's split of each unit into partial
 * sums, so outputs may differ from the default in their last bits. */
NOSA_API nosa_status nosa_create(const nosa_config* cfg, nosa_ctx** out);

/* Free everything nosa_create allocated (synchronises the device first).
 * NULL is ignored. */
NOSA_API void nosa_destroy(nosa_ctx* ctx);

/* Attach the KV of every unit and reset the decode state (step 0, cold cache).
 * k, v: bf16 [U, max_blocks*P, d] row-major (unit, token, dim).  With
 *   cache_slots > 0 they must be pinned host memory: the full cache lives on the
 *   host (NOSA summary §1, §4) and blocks closed during decoding are written
 *   through into it.  With cache_slots = 0 they are device memory.
 *   Base addresses must be 16-byte aligned.
 * n_tokens: prompt tokens per unit, k*P <= n_tokens <= max_blocks*P.  Tokens
 *   beyond the last full block become the open tail block.
 * agnostic: device fp32 [U, max_blocks], the query-agnostic score of every
 *   block (copied; entries of blocks that close later are replaced by
 *   nosa_append_token's value).
 * Builds the pooled keys (one read of K; over PCIe when offloaded) on stream.
 */
NOSA_API nosa_status nosa_attach_kv(nosa_ctx* ctx, const void* k, const void* v, int n_tokens,
                           const float* agnostic, nosa_stream_t stream);

/* Append one token per unit to the open tail block (first call of a step).
 * NOSA summary App. A describes one decode step over a context that grows by
 * the token just decoded; the reading here is that its K/V join an open tail
 * block that is attended in full but neither scored nor fetched until its 64
 * tokens close it, after which it is an ordinary candidate block (pooled keys
 * as in §3.1, agnostic score as passed, stored on the host as in §1).
 * k_new, v_new: device bf16 [B, H_kv, d].  agnostic_if_close: device fp32 [U]
 * or NULL; it becomes the agnostic score of the tail block if this token fills
 * it, in which case nosa_sparse_decode closes the block at the end of the step
 * (pooled keys built, candidate from the next step on).  A closed block's K/V
 * reach the attached KV at once when it is device memory.  When it is host
 * memory they are staged in HBM and written through while the next step runs
 * (a low-priority kernel on a stream of the context, forked by
 * nosa_score_blocks and joined by nosa_sparse_decode); until then the miss
 * gather reads the staged copy.  nosa_get_state, nosa_set_state and
 * nosa_attach_kv land a pending write-through first, so after a step the host
 * copy of the last closed block is complete once the next step has run or one
 * of those calls has returned.
 * NOSA_ERR_INVALID when the unit would exceed max_blocks*P tokens. */
NOSA_API nosa_status nosa_append_token(nosa_ctx* ctx, const void* k_new, const void* v_new,
                              const float* agnostic_if_close, nosa_stream_t stream);

/* Two-stage block scores (NOSA summary §3.1): for each unit and closed block j,
 *   scores[u*max_blocks + j] = max_{r<R} sum_{h in group(u)} q_h . kbar[u, j*R + r]
 * where kbar is the mean of each sub-block's 16 keys rounded once to bf16.
 * Products are exact and sums are fp64.  q: device bf16 [B, H_q, d].
 * scores: device fp64 [U, max_blocks]; entries j >= n are left untouched. */
NOSA_API nosa_status nosa_score_blocks(nosa_ctx* ctx, const void* q, double* scores, nosa_stream_t stream);

/* Selection (NOSA summary §2.1, §3.1, App. B.2.2, App. E), per unit, with
 * F(t) the forced blocks (first sink_blocks and last window_blocks closed):
 *   Gamma_e(t) = top-(k_e - |F|) by agnostic score of Gamma_e(t-1) plus the
 *                blocks that became eligible (closed outside the window, or
 *                slid out of it) since the last step (all eligible blocks at
 *                step 0); an evicted block never re-enters Gamma_e.
 *   c_t        = max(0, (k - m) - |(F ∪ Gamma_e)(t) \ S(t-1)|)   (no cap at step 0)
 *   Gamma_q(t) = top-k_q by score of (S(t-1) \ (F ∪ Gamma_e)(t)) ∪ top-c_t of
 *                the blocks in neither (F ∪ Gamma_e)(t) nor S(t-1)
 *   S(t)       = F(t) ∪ Gamma_e(t) ∪ Gamma_q(t)
 * Ties go to the lower block id.  scores: device fp64 as written by
 * nosa_score_blocks.  sel: device int32 [U, k], S(t) ascending, -1 padded. */
NOSA_API nosa_status nosa_select(nosa_ctx* ctx, const double* scores, int32_t* sel, nosa_stream_t stream);

/* Cache planning (NOSA summary §4, App. A).  This call plans only: it moves
 * no bytes, and when its stream has drained the missed blocks are still in
 * host memory; nosa_sparse_decode copies them.  Per unit the
 * misses M = S(t) \ R(t-1) (R = blocks resident in the GPU cache) get slots:
 * free slots first (lowest first), then resident blocks outside S(t), least
 * recently selected first, lower block id on ties.  Only blocks unused by this
 * step are replaced.  sel: device int32 [U, k] from nosa_select.  fetch:
 * device int32 [U, k], the missed block ids ascending, -1 padded.  n_fetch:
 * device int32 [U].  Planning runs on compute, and the slot tables
 * (nosa_read_cache_map) are final when it has run.  The copies themselves --
 * K and V of each miss, 2 x 16 KiB, from pinned host memory into its slot by
 * a zero-copy gather kernel that also attends to each block as it lands --
 * are issued by nosa_sparse_decode on its stream.  `copy` names a second
 * stream (it may equal compute): when it differs, nosa_sparse_decode runs the
 * attention to the blocks already cached on it, beside the transfer, and
 * joins it back.  With KV resident (cache_slots = 0) nothing is copied:
 * fetch is all -1 and n_fetch all 0. */
NOSA_API nosa_status nosa_fetch_missing(nosa_ctx* ctx, const int32_t* sel, int32_t* fetch,
                               int32_t* n_fetch, nosa_stream_t compute, nosa_stream_t copy);

/* nosa_score_blocks, nosa_select and nosa_fetch_missing in one call, with
 * the same arguments, results and order rule (first call of a step, after an
 * optional nosa_append_token); on return the step is ready for
 * nosa_sparse_decode.  With max_blocks <= 512 the scores, the selection and
 * the cache plan of each unit come from one kernel (one CTA per unit), so the
 * miss gather starts after a single launch; scores, sel, fetch and n_fetch
 * are bit-identical to those of the three calls.  With more blocks it makes
 * the three calls itself. */
NOSA_API nosa_status nosa_score_select_fetch(nosa_ctx* ctx, const void* q, double* scores, int32_t* sel,
                                             int32_t* fetch, int32_t* n_fetch, nosa_stream_t compute,
                                             nosa_stream_t copy);

/* One whole decode step in one call (NOSA summary App. A: select, move the
 * missed blocks CPU -> GPU, attend): nosa_score_select_fetch followed by
 * nosa_sparse_decode, with the same results bit for bit.  q (bf16
 * [B, H_q, d]) and out (bf16 [B, H_q, d]) may each be device memory or pinned
 * host memory, 16-byte aligned.  Queries in host memory are read over PCIe
 * once, by the kernel that scores the blocks (up to 512 blocks per unit; with
 * more, by one copy at the start of the step), and kept in a device copy for
 * the attention; outputs to host memory are written there directly by the
 * kernels that finish each unit.  So a decode loop whose queries and outputs
 * live on the host needs no copies of its own and no wait per step: out is
 * complete once `compute` has reached the end of the step.
 * scores, sel, fetch, n_fetch: as in nosa_score_select_fetch (device), or
 * NULL to use buffers of the context.  Same order rule as
 * nosa_score_select_fetch (after an optional nosa_append_token). */
NOSA_API nosa_status nosa_decode_step(nosa_ctx* ctx, const void* q, double* scores, int32_t* sel, int32_t* fetch,
                                      int32_t* n_fetch, void* out, nosa_stream_t compute, nosa_stream_t copy);

/* Block-sparse GQA attention (NOSA summary App. A): for each query head h of
 * unit u,  out_h = sum_t softmax_t(q_h . K_t / sqrt(d)) V_t  over the tokens of
 * the selected blocks plus the open tail, in fp32 with bf16 inputs; written as
 * bf16.  q: device bf16 [B, H_q, d]; sel: the same buffer passed to
 * nosa_select; out: device bf16 [B, H_q, d].  With KV in host memory it also
 * issues the miss gather planned by the fetch call, on `stream`, and -- when
 * the fetch call was given a second stream -- runs the attention to the
 * cached blocks on that stream beside it (joined back into `stream` before
 * it returns).  Ends the step: closes a full tail block and advances the step
 * counter. */
NOSA_API nosa_status nosa_sparse_decode(nosa_ctx* ctx, const void* q, const int32_t* sel, void* out,
                               nosa_stream_t stream);

/* Allocation-free variant of the attention step (no counterpart on the
 * pages: it exists for embedders).  Some callers cannot call cudaMalloc: a
 * serving engine that reserves nearly all of HBM for its own pool allocator
 * leaves no room for a library's private buffers, and code that must not add
 * device-wide synchronisation (cudaMalloc / cudaFree may synchronise) cannot
 * create a context.  This call needs no context and allocates nothing.
 *
 * It computes what nosa_sparse_decode computes for resident KV without a tail:
 * for each query head h of unit u, out_h = softmax(q_h K^T / sqrt(d)) V over the
 * 64 tokens of each block listed in sel[u].  q: device bf16 [B, H_q, 128];
 * k, v: device bf16 [U, max_blocks*64, 128], 16-byte aligned; sel: device
 * int32 [U, k_sel] of block ids (an out-of-range id is flagged and block 0 is
 * read in its place); out: device bf16 [B, H_q, 128].  With the same inputs the
 * output is bit-identical to nosa_sparse_decode's over resident KV.  Split-KV
 * partials live in a fixed array inside the library (8.5 MB per GPU that loads
 * it, held until exit): the call returns NOSA_ERR_INVALID when B*H_q exceeds
 * 8192 query heads.
 * The first call on a device resolves that array's device address (once per
 * device, with the device current), so make it before any stream capture.
 * Every call shares the array and leaves its contents behind; each call
 * clears the merge counters it needs and fully writes the partials it reads,
 * but calls that overlap on the GPU (on different streams) race.  Device-side
 * errors (an out-of-range id, a bounded wait that ran out and left outputs
 * unwritten) are not returned by this asynchronous call: they accumulate in a
 * per-device error word that nosa_noalloc_check_errors reports. */
NOSA_API nosa_status nosa_sparse_decode_noalloc(const void* q, const void* k, const void* v, int batch,
                                                int n_q_heads, int n_kv_heads, int max_blocks,
                                                const int32_t* sel, int k_sel, void* out,
                                                nosa_stream_t stream);

/* Synchronous (waits for stream).  Reports and clears the error word that
 * nosa_sparse_decode_noalloc calls on the current device have set since the
 * last check: NOSA_ERR_TIMEOUT when a bounded device wait ran out (that call's
 * outputs are incomplete), NOSA_ERR_INVALID when a selected block id was out of
 * range, else NOSA_OK.  Allocates nothing. */
NOSA_API nosa_status nosa_noalloc_check_errors(nosa_stream_t stream);

/* Row gather at a chosen granularity (NOSA summary §3.2 and §4: block-wise
 * transfer of 16 KiB blocks against element-wise transfer of single tokens).
 * For i < n: row dst_idx[i] of dst  <-  row src_idx[i] of src, each row
 * row_bytes long (a power of two in [16, 65536]); dst_idx = NULL means row i.
 * A miss of the decode step is two 16 KiB rows (its K and its V block); a
 * token is two 256-byte rows at d = 128, bf16.
 * src: device-addressable memory of src_rows rows (pinned host memory mapped
 * into the device's address space, or device memory); dst: device memory of
 * dst_rows rows; both 16-byte aligned.  src_idx, dst_idx: device int64 [n].
 * ctas: CTAs of 256 threads, 0 for a quarter of the SMs (the decode step's
 * gather width).  flags: device uint32 or NULL; bit 0 is ORed in when an
 * index is out of range, and that row is skipped.  Destination rows must be
 * distinct (two copies into one row race).  Asynchronous on stream; n = 0
 * launches nothing.  NOSA_ERR_INVALID for bad sizes, NULL pointers, a src the
 * device cannot address (pageable host memory) or a dst, index or flags
 * pointer that is not device memory. */
NOSA_API nosa_status nosa_gather_rows(const void* src, int64_t src_rows, void* dst, int64_t dst_rows,
                                      int32_t row_bytes, const int64_t* src_idx, const int64_t* dst_idx,
                                      int32_t n, int32_t ctas, uint32_t* flags, nosa_stream_t stream);

/* The row gather of nosa_gather_rows (same arguments, result and errors)
 * through the TMA unit instead of SM loads: every row, or 16 KiB piece of a
 * longer row, is one asynchronous bulk copy into shared memory (completing
 * on an mbarrier) and one bulk copy out to dst.  It is the transfer study's
 * second arm (NOSA summary §4: a dedicated transfer kernel over 16 KiB blocks
 * through unified virtual addressing): the bulk copies issue their own PCIe
 * read requests.  ctas: CTAs of 4 copying warps, 0 for a quarter of the SMs.
 * flags bit 1 is ORed in when a copy did not complete within about 1 s (the
 * kernel stops early; the context of the caller stays usable). */
NOSA_API nosa_status nosa_gather_rows_bulk(const void* src, int64_t src_rows, void* dst, int64_t dst_rows,
                                           int32_t row_bytes, const int64_t* src_idx, const int64_t* dst_idx,
                                           int32_t n, int32_t ctas, uint32_t* flags, nosa_stream_t stream);

/* Synchronous.  Copies the running totals into *stats. */
NOSA_API nosa_status nosa_get_stats(nosa_ctx* ctx, nosa_stats* stats);

/* Zero the running totals (asynchronous on stream). */
NOSA_API nosa_status nosa_reset_stats(nosa_ctx* ctx, nosa_stream_t stream);

/* Synchronous.  NOSA_ERR_TIMEOUT if a bounded device wait ran out,
 * NOSA_ERR_INVALID if a device-side bounds or capacity check fired, else
 * NOSA_OK.  Bits: 1 wait timeout, 2 append beyond capacity, 4 cache planning
 * found no slot, 8 gather or decode index out of range. */
NOSA_API nosa_status nosa_check_errors(nosa_ctx* ctx);

/* Synchronous.  Host int32 [U, cache_slots]: the block held by each cache
 * slot, -1 if free.  NOSA_ERR_INVALID when KV is resident. */
NOSA_API nosa_status nosa_read_cache_map(nosa_ctx* ctx, int32_t* slot_block);

/* Synchronous.  Copies the GPU block cache of units [unit_begin,
 * unit_begin + n_units) into host buffers k_host, v_host, each bf16
 * [n_units, cache_slots, P, d]: slot s of a unit holds the K (V) rows of the
 * block nosa_read_cache_map names for it (contents of free slots are
 * unspecified).  For checking the miss gather (NOSA summary §4: the missed
 * blocks land in their GPU slots).  NOSA_ERR_INVALID when KV is resident or
 * the range is outside [0, U). */
NOSA_API nosa_status nosa_read_cache(nosa_ctx* ctx, int unit_begin, int n_units, void* k_host, void* v_host);

/* Synchronous checkpoint of the decode state: step counter, block count,
 * Gamma_e, S(t-1), cache tables, agnostic scores and the open tail block.
 * Pass buf = NULL to query the size in *size.  Cache contents and pooled keys
 * are not stored: nosa_set_state rebuilds them from the attached KV. */
NOSA_API nosa_status nosa_get_state(nosa_ctx* ctx, void* buf, size_t* size);

/* Synchronous restore of a nosa_get_state blob taken from a context with the
 * same config and attached KV.  Rebuilds pooled keys and refills the cache. */
NOSA_API nosa_status nosa_set_state(nosa_ctx* ctx, const void* buf, size_t size);

/* Diagnostic: enqueue a kernel that waits until *flag (device or pinned host
 * int32) becomes nonzero or timeout_ms elapses; on timeout it sets error bit 1
 * and returns, leaving the context usable. */
NOSA_API nosa_status nosa_debug_wait_flag(nosa_ctx* ctx, const int32_t* flag, int timeout_ms,
                                 nosa_stream_t stream);

/* Diagnostic: inject one host-side CUDA failure on the calling thread.  The
 * context calls (nosa_create ... nosa_set_state) check every CUDA runtime call
 * they make; after this call the check that follows `skip` further checks is
 * not made at all and reports cudaErrorLaunchFailure instead, so that call
 * returns NOSA_ERR_CUDA.  Nothing reaches the GPU.  The work the failed call
 * enqueued before the failure still runs; nosa_attach_kv brings the context
 * back to a clean step 0.  skip = -1 cancels a pending injection. */
NOSA_API nosa_status nosa_debug_inject_cuda_error(int skip);

/* Message of the last failure on the calling thread ("" if none). */
NOSA_API const char* nosa_last_error(void);

/* Library version string. */
NOSA_API const char* nosa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NOSA_H */
