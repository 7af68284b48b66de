/*
 * nosa_oracle.c -- TEST INFRASTRUCTURE, NOT PRODUCT CODE.
 *
 * A plain, slow, fp64 CPU restatement of one NOSA decode step, written from the
 * pages that describe the method.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline / reference arm may build, load or call it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Sources (page title, section):
 *  [S31]  NOSA: Native and Offloadable Sparse Attention (paperlayer summary), §3.1
 *         -- minimum overlap gamma0 between adjacent steps; budget split into a
 *         query-aware and a query-agnostic subset; two-stage block scoring with
 *         mean pooling over sub-blocks then max pooling to the block.
 *  [S21]  same page, §2.1 -- query-aware top-k vs query-agnostic eviction.
 *  [S22]  same page, §2.2 -- locality: the share of step t's selected tokens
 *         that step t-1 had selected too.
 *  [S4]   same page, §4 -- a kernel compares the old and new selections and
 *         decides which cached blocks give up their slots; blocks the step
 *         uses keep theirs; cached blocks need not sit contiguously.
 *  [SA]   same page, App. A (pseudocode summary) -- per step: select blocks,
 *         transfer the cache-missed blocks CPU->GPU, attend with the cache.
 *  [SE]   same page, App. E -- |Gamma(t-1) ∩ Gamma(t)| >= k_e.
 *  [GX]   NOSA: Native and Offloadable Sparse Attention (gist.science explainer),
 *         technical summary, "Method / 1. Algorithm" -- the eviction rule (a unit
 *         not selected at step t is never selected again by the query-agnostic
 *         part), gamma(t) >= k_e/k, and the pooling order (mean within sub-blocks,
 *         then max at block level).
 *
 * Where the pages leave a step open, the plainest reading is taken; each such
 * reading is named at the function that implements it.
 *
 * Parity status: every function here is pinned by CPU tests against closed
 * forms, brute force on tiny inputs or invariants; none has a printed worked
 * example on the pages.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp64                                                             */
/* ------------------------------------------------------------------------ */

double orc_bf16_to_f64(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round an fp64 value to the nearest bf16 value, ties to even.  bf16 keeps 8
 * significant bits with fp32's exponent range; below 2^-126 the grid spacing is
 * fixed at 2^-133.  E = max(floor(log2|x|), -126) picks the grid spacing
 * 2^(E-7); r = rint(|x| / 2^(E-7)) is the rounded significand (rint rounds half
 * to even); the encoding is ((E + 126) << 7) + r, which carries into the
 * exponent when r reaches 256 and yields subnormal encodings when E = -126. */
uint16_t orc_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7F80);
  int e2;
  frexp(a, &e2);            /* a = f * 2^e2, f in [0.5, 1) */
  int E = e2 - 1;           /* floor(log2 a) */
  if (E < -126) E = -126;
  double r = nearbyint(ldexp(a, 7 - E));
  long bits = ((long)(E + 126) << 7) + (long)r;
  if (bits >= 0x7F80) bits = 0x7F80;
  return (uint16_t)(sign | (uint16_t)bits);
}

/* ------------------------------------------------------------------------ */
/* a0: pooled keys [S31][GX] -- mean over each sub-block of Q tokens.          */
/* ------------------------------------------------------------------------ */

/* K: bf16 [n_sub * Q][d]; kbar: bf16 [n_sub][d].
 * kbar[s][i] = bf16( (sum_{j<Q} K[s*Q + j][i]) / Q ), the sum taken in fp64. */
void orc_pool_keys(const uint16_t* K, int n_sub, int Q, int d, uint16_t* kbar) {
  for (int s = 0; s < n_sub; ++s) {
    for (int i = 0; i < d; ++i) {
      double sum = 0.0;
      for (int j = 0; j < Q; ++j) sum += orc_bf16_to_f64(K[(size_t)(s * Q + j) * d + i]);
      kbar[(size_t)s * d + i] = orc_f64_to_bf16(sum / (double)Q);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* a1: block scores [S31][GX] -- query vs pooled sub-block keys, then the max  */
/* over the sub-blocks of a block.                                            */
/* ------------------------------------------------------------------------ */

/* Reading (group aggregation): a KV head serves G query heads; the sub-block
 * score is the sum over those heads of the raw dot products q_h . kbar_s (no
 * softmax, no 1/sqrt(d): neither changes the ordering of a single head, and
 * summing the raw products is the plainest aggregate).
 * q: bf16 [G][d]; kbar: bf16 [n_blocks * R][d]; score: fp64 [n_blocks]. */
void orc_score_blocks(const uint16_t* q, int G, int d, const uint16_t* kbar,
                      int n_blocks, int R, double* score) {
  for (int j = 0; j < n_blocks; ++j) {
    double best = -INFINITY;
    for (int r = 0; r < R; ++r) {
      const uint16_t* kb = kbar + (size_t)(j * R + r) * d;
      double s = 0.0;
      for (int h = 0; h < G; ++h)
        for (int i = 0; i < d; ++i)
          s += orc_bf16_to_f64(q[h * d + i]) * orc_bf16_to_f64(kb[i]);
      if (s > best) best = s;
    }
    score[j] = best;
  }
}

/* ------------------------------------------------------------------------ */
/* Orderings.                                                                */
/* Reading (ties): larger score first; equal scores go to the lower block id. */
/* ------------------------------------------------------------------------ */

typedef struct { double key; int idx; } orc_item;

static int orc_item_cmp(const void* pa, const void* pb) {
  const orc_item* a = (const orc_item*)pa;
  const orc_item* b = (const orc_item*)pb;
  if (a->key > b->key) return -1;
  if (a->key < b->key) return 1;
  return (a->idx > b->idx) - (a->idx < b->idx);
}

static int orc_int_cmp(const void* pa, const void* pb) {
  int a = *(const int*)pa, b = *(const int*)pb;
  return (a > b) - (a < b);
}

/* ------------------------------------------------------------------------ */
/* a2: query-agnostic set with eviction [S21][GX].                            */
/* ------------------------------------------------------------------------ */

/* The query-agnostic part keeps at most k_e blocks ranked by their agnostic
 * score a[j].  Eviction rule: a block that is not in Gamma_e(t) can never be in
 * Gamma_e(t') for t' > t.  Reading: the only blocks that may join are those
 * that closed since the previous step, so the pool is
 *   Gamma_e(t-1) ∪ { j : n_from <= j < n_to }
 * and Gamma_e(t) is its top-k_e by (a desc, id asc).  At the first step the
 * pool is every closed block (caller passes n_ge_prev = 0, n_from = 0).
 * ge_out is written in ascending block order; returns |Gamma_e(t)|. */
int orc_evict_update(const float* a, const int* ge_prev, int n_ge_prev, int n_from,
                     int n_to, int k_e, int* ge_out) {
  int pool_n = n_ge_prev + (n_to > n_from ? n_to - n_from : 0);
  orc_item* pool = (orc_item*)malloc(sizeof(orc_item) * (size_t)(pool_n > 0 ? pool_n : 1));
  int p = 0;
  for (int i = 0; i < n_ge_prev; ++i) { pool[p].key = (double)a[ge_prev[i]]; pool[p].idx = ge_prev[i]; ++p; }
  for (int j = n_from; j < n_to; ++j) { pool[p].key = (double)a[j]; pool[p].idx = j; ++p; }
  qsort(pool, (size_t)p, sizeof(orc_item), orc_item_cmp);
  int take = p < k_e ? p : k_e;
  for (int i = 0; i < take; ++i) ge_out[i] = pool[i].idx;
  qsort(ge_out, (size_t)take, sizeof(int), orc_int_cmp);
  free(pool);
  return take;
}

/* ------------------------------------------------------------------------ */
/* a3: query-aware selection under the minimum-overlap constraint [S31][SE].   */
/* ------------------------------------------------------------------------ */

/* S(t) = F(t) ∪ Gamma_e(t) ∪ Gamma_q(t).  F(t) is the set of forced blocks
 * (attention sink and sliding window, see orc_forced; empty unless
 * configured).  Gamma_q(t) is drawn from blocks outside F(t) ∪ Gamma_e(t)
 * (the budget is divided between the subsets).
 * Reading (gamma0): at most c_max = k - m blocks of S(t) may be absent from
 * S(t-1).  Forced and query-agnostic blocks that are new use that allowance
 * first:
 *   c_t = max(0, c_max - |(F(t) ∪ Gamma_e(t)) \ S(t-1)|)
 *   O   = S(t-1) \ (F(t) ∪ Gamma_e(t))             (old candidates)
 *   N   = blocks outside F(t) ∪ Gamma_e(t) ∪ S(t-1)  (new candidates)
 *   Gamma_q(t) = top-k_q of ( O ∪ top-c_t(N) )      by (score desc, id asc)
 * At the first step S(-1) is empty and there is no cap: Gamma_q(0) is the
 * top-k_q of every block outside F(0) ∪ Gamma_e(0).
 * forced: n flags (NULL = none).  sel_out gets S(t) ascending; returns |S(t)|. */
int orc_select_forced(const double* score, int n, const unsigned char* forced, const int* ge, int n_ge,
                      const int* prev, int n_prev, int first, int k_q, int c_max, int* sel_out) {
  unsigned char* in_e = (unsigned char*)calloc((size_t)n + 1, 1);  /* F ∪ Gamma_e */
  unsigned char* in_p = (unsigned char*)calloc((size_t)n + 1, 1);
  orc_item* cand = (orc_item*)malloc(sizeof(orc_item) * (size_t)(n + 1));
  orc_item* newc = (orc_item*)malloc(sizeof(orc_item) * (size_t)(n + 1));
  for (int i = 0; i < n_ge; ++i) in_e[ge[i]] = 1;
  if (forced) for (int j = 0; j < n; ++j) if (forced[j]) in_e[j] = 1;
  for (int i = 0; i < n_prev; ++i) if (prev[i] < n) in_p[prev[i]] = 1;

  int nc = 0;
  if (first) {
    for (int j = 0; j < n; ++j)
      if (!in_e[j]) { cand[nc].key = score[j]; cand[nc].idx = j; ++nc; }
  } else {
    int e_new = 0;
    for (int j = 0; j < n; ++j) if (in_e[j] && !in_p[j]) ++e_new;
    int c_t = c_max - e_new;
    if (c_t < 0) c_t = 0;
    int nn = 0;
    for (int j = 0; j < n; ++j) {
      if (in_e[j]) continue;
      if (in_p[j]) { cand[nc].key = score[j]; cand[nc].idx = j; ++nc; }
      else { newc[nn].key = score[j]; newc[nn].idx = j; ++nn; }
    }
    qsort(newc, (size_t)nn, sizeof(orc_item), orc_item_cmp);
    for (int i = 0; i < nn && i < c_t; ++i) cand[nc++] = newc[i];
  }
  qsort(cand, (size_t)nc, sizeof(orc_item), orc_item_cmp);
  int nq = nc < k_q ? nc : k_q;

  int ns = 0;
  for (int j = 0; j < n; ++j) if (in_e[j]) sel_out[ns++] = j;
  for (int i = 0; i < nq; ++i) sel_out[ns++] = cand[i].idx;
  qsort(sel_out, (size_t)ns, sizeof(int), orc_int_cmp);
  free(in_e); free(in_p); free(cand); free(newc);
  return ns;
}

/* The selection without forced blocks. */
int orc_select(const double* score, int n, const int* ge, int n_ge, const int* prev,
               int n_prev, int first, int k_q, int c_max, int* sel_out) {
  return orc_select_forced(score, n, NULL, ge, n_ge, prev, n_prev, first, k_q, c_max, sel_out);
}

/* Forced blocks (NOSA: Native and Offloadable Sparse Attention, paperlayer
 * summary, App. B.2.2: one attention-sink block and 16 sliding-window blocks,
 * counted inside the 48 query-agnostic blocks of NOSA's budget, and the same
 * sink and window for InfLLMv2).  Reading: the sink is the first `sink`
 * closed blocks, the window the last `window` closed blocks.  Flags n entries;
 * returns how many are forced. */
int orc_forced(int n, int sink, int window, unsigned char* is_forced) {
  int c = 0;
  for (int j = 0; j < n; ++j) {
    is_forced[j] = (unsigned char)(j < sink || j >= n - window);
    c += is_forced[j];
  }
  return c;
}

/* ------------------------------------------------------------------------ */
/* a4: cache bookkeeping -- set difference and replacement mapping [S4][SA].   */
/* ------------------------------------------------------------------------ */

typedef struct { long key1; int key2; int slot; } orc_victim;

static int orc_victim_cmp(const void* pa, const void* pb) {
  const orc_victim* a = (const orc_victim*)pa;
  const orc_victim* b = (const orc_victim*)pb;
  if (a->key1 != b->key1) return (a->key1 > b->key1) - (a->key1 < b->key1);
  return (a->key2 > b->key2) - (a->key2 < b->key2);
}

/* The GPU cache holds C block slots per unit; slot_block[c] is the block in
 * slot c or -1, last_used[c] the last step that selected it.
 * Misses M = S(t) \ R(t-1), in ascending block order, are what must cross
 * PCIe.  Only blocks unused by the current step may be replaced.
 * Reading (replacement order): free slots go first, lowest slot first; then
 * resident blocks outside S(t), least recently selected first, lower block id
 * on ties.  The i-th miss takes the i-th slot of that order.  Hits and
 * inserted blocks get last_used = step.
 * fetch[i] = i-th missed block, fetch_slot[i] its slot; returns |M|, or -1 if
 * the cache cannot hold S(t) (fewer than |S(t)| slots). */
int orc_cache_plan(const int* sel, int ns, int step, int C, int* slot_block,
                   int* last_used, int* fetch, int* fetch_slot) {
  int nm = 0;
  for (int i = 0; i < ns; ++i) {
    int hit = -1;
    for (int c = 0; c < C; ++c) if (slot_block[c] == sel[i]) { hit = c; break; }
    if (hit >= 0) last_used[hit] = step;
    else fetch[nm++] = sel[i];
  }
  if (nm == 0) return 0;

  int* order = (int*)malloc(sizeof(int) * (size_t)C);
  orc_victim* vic = (orc_victim*)malloc(sizeof(orc_victim) * (size_t)C);
  int no = 0, nv = 0;
  for (int c = 0; c < C; ++c) if (slot_block[c] < 0) order[no++] = c;
  for (int c = 0; c < C; ++c) {
    if (slot_block[c] < 0) continue;
    int selected = 0;
    for (int i = 0; i < ns; ++i) if (sel[i] == slot_block[c]) { selected = 1; break; }
    if (selected) continue;
    vic[nv].key1 = last_used[c]; vic[nv].key2 = slot_block[c]; vic[nv].slot = c; ++nv;
  }
  qsort(vic, (size_t)nv, sizeof(orc_victim), orc_victim_cmp);
  for (int i = 0; i < nv; ++i) order[no++] = vic[i].slot;
  if (no < nm) { free(order); free(vic); return -1; }
  for (int i = 0; i < nm; ++i) {
    int c = order[i];
    slot_block[c] = fetch[i];
    last_used[c] = step;
    fetch_slot[i] = c;
  }
  free(order); free(vic);
  return nm;
}

/* ------------------------------------------------------------------------ */
/* a6: attention over the selected tokens [SA].                               */
/* ------------------------------------------------------------------------ */

/* For each query head h: o_h = sum_t softmax_t(q_h . K_t / sqrt(d)) V_t over
 * the given token rows, in fp64 with the max subtracted before exp.
 * q: bf16 [G][d]; K, V: bf16 [*][d] (the unit's token rows); rows: token ids;
 * out: fp64 [G][d]. */
void orc_attend(const uint16_t* q, int G, int d, const uint16_t* K, const uint16_t* V,
                const int* rows, int n_rows, double* out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1));
  double scale = 1.0 / sqrt((double)d);
  for (int h = 0; h < G; ++h) {
    double mx = -INFINITY;
    for (int t = 0; t < n_rows; ++t) {
      const uint16_t* kr = K + (size_t)rows[t] * d;
      double dot = 0.0;
      for (int i = 0; i < d; ++i) dot += orc_bf16_to_f64(q[h * d + i]) * orc_bf16_to_f64(kr[i]);
      s[t] = dot * scale;
      if (s[t] > mx) mx = s[t];
    }
    double den = 0.0;
    for (int t = 0; t < n_rows; ++t) { s[t] = exp(s[t] - mx); den += s[t]; }
    for (int i = 0; i < d; ++i) {
      double num = 0.0;
      for (int t = 0; t < n_rows; ++t) num += s[t] * orc_bf16_to_f64(V[(size_t)rows[t] * d + i]);
      out[h * d + i] = num / den;
    }
  }
  free(s);
}

/* ------------------------------------------------------------------------ */
/* Whole decode trajectory of one unit (one sequence, one KV head).           */
/* ------------------------------------------------------------------------ */

typedef struct {
  int G, d, P, Q;        /* group size, head dim, block, sub-block */
  int n0, tail0;         /* closed blocks and tail tokens at attach */
  int max_blocks;        /* capacity of K/V/a in blocks */
  int k_q, k_e, m;       /* budget split and minimum overlap */
  int C;                 /* cache slots; 0 = KV resident on the GPU */
  int steps;
  int append;            /* 1: one token appended per step */
  int sink, window;      /* forced blocks, counted inside k_e (0, 0 = none) */
} orc_cfg;

/* Per step t, in this order:
 *   append (token n*P + tail goes into the open tail block) ->
 *   pooled keys of newly closed blocks -> scores -> Gamma_e update ->
 *   capped query-aware selection -> cache plan (offloaded) ->
 *   attention over S(t) plus the open tail -> close the tail if it is full.
 * Reading (tail): the open tail block is always attended, never scored, never
 * fetched; a block that closes at step t becomes a candidate from t+1 on and is
 * not inserted into the cache.
 * Inputs: K, V bf16 [max_blocks*P][d] (rows beyond the prompt are the tokens
 * appended during decoding); a fp32 [max_blocks]; q bf16 [steps][G][d];
 * attend_mask[t] != 0 requests the attention output of step t.
 * Outputs (may be NULL): sel [steps][k] (-1 pad), nsel [steps],
 * fetch [steps][k] (-1 pad), nfetch [steps], resident [steps][C] (sorted
 * block ids, -1 pad), o fp64 [steps][G][d], overlap [steps] = |S(t) ∩ S(t-1)|,
 * scores fp64 [steps][max_blocks] (NaN beyond n).
 * Returns 0, or a negative code on bad input. */
int orc_run_unit(const orc_cfg* cfg, const uint16_t* K, const uint16_t* V, const float* a,
                 const uint16_t* q, const unsigned char* attend_mask,
                 int* out_sel, int* out_nsel, int* out_fetch, int* out_nfetch,
                 int* out_resident, double* out_o, int* out_overlap, double* out_scores) {
  const int G = cfg->G, d = cfg->d, P = cfg->P, Q = cfg->Q, R = P / Q;
  const int k = cfg->k_q + cfg->k_e, c_max = k - cfg->m, C = cfg->C;
  const int k_e_dyn = cfg->k_e - cfg->sink - cfg->window;  /* agnostic blocks beyond the forced ones */
  if (P % Q != 0 || k <= 0 || cfg->m > k || cfg->n0 > cfg->max_blocks) return -1;
  if (k_e_dyn < 0 || cfg->sink < 0 || cfg->window < 0) return -1;
  if (C > 0 && C < k) return -2;

  uint16_t* kbar = (uint16_t*)calloc((size_t)cfg->max_blocks * R * d, sizeof(uint16_t));
  double* score = (double*)malloc(sizeof(double) * (size_t)(cfg->max_blocks + 1));
  int* ge = (int*)malloc(sizeof(int) * (size_t)(cfg->k_e + 1));
  int* ge_new = (int*)malloc(sizeof(int) * (size_t)(cfg->k_e + 1));
  int* prev = (int*)malloc(sizeof(int) * (size_t)(k + 1));
  int* sel = (int*)malloc(sizeof(int) * (size_t)(k + cfg->k_e + 1));
  int* slot_block = (int*)malloc(sizeof(int) * (size_t)(C + 1));
  int* last_used = (int*)malloc(sizeof(int) * (size_t)(C + 1));
  int* fetch = (int*)malloc(sizeof(int) * (size_t)(k + 1));
  int* fetch_slot = (int*)malloc(sizeof(int) * (size_t)(k + 1));
  int* rows = (int*)malloc(sizeof(int) * (size_t)(k * P + P + 1));
  unsigned char* forced = (unsigned char*)calloc((size_t)cfg->max_blocks + 1, 1);
  for (int c = 0; c < C; ++c) { slot_block[c] = -1; last_used[c] = -1; }

  int n = cfg->n0, tail = cfg->tail0, n_ge = 0, n_prev = 0, n_at_last_select = 0, rc = 0;
  orc_pool_keys(K, n * R, Q, d, kbar);

  for (int t = 0; t < cfg->steps; ++t) {
    if (cfg->append) {
      if (n * P + tail >= cfg->max_blocks * P) { rc = -3; break; }
      tail += 1;
    }
    orc_score_blocks(q + (size_t)t * G * d, G, d, kbar, n, R, score);
    if (out_scores) {
      for (int j = 0; j < cfg->max_blocks; ++j)
        out_scores[(size_t)t * cfg->max_blocks + j] = j < n ? score[j] : NAN;
    }
    int first = (t == 0);
    /* Eligible for Gamma_e: closed blocks outside the sink and the window,
     * [sink, n - window).  Blocks that became eligible since the last step
     * (closed there, or slid out of the window) join its pool. */
    orc_forced(n, cfg->sink, cfg->window, forced);
    int e_to = n - cfg->window;
    int e_from = first ? cfg->sink : n_at_last_select - cfg->window;
    if (e_from < cfg->sink) e_from = cfg->sink;
    if (e_to < e_from) e_to = e_from;
    int n_e = orc_evict_update(a, ge, first ? 0 : n_ge, e_from, e_to, k_e_dyn, ge_new);
    memcpy(ge, ge_new, sizeof(int) * (size_t)n_e);
    n_ge = n_e;
    n_at_last_select = n;
    int ns = orc_select_forced(score, n, forced, ge, n_ge, prev, n_prev, first, cfg->k_q, c_max, sel);

    int ov = 0;
    for (int i = 0; i < ns; ++i)
      for (int j = 0; j < n_prev; ++j) if (prev[j] == sel[i]) { ++ov; break; }
    if (out_overlap) out_overlap[t] = ov;
    if (out_sel) for (int i = 0; i < k; ++i) out_sel[(size_t)t * k + i] = i < ns ? sel[i] : -1;
    if (out_nsel) out_nsel[t] = ns;

    if (C > 0) {
      int nf = orc_cache_plan(sel, ns, t, C, slot_block, last_used, fetch, fetch_slot);
      if (nf < 0) { rc = -4; break; }
      if (out_fetch) for (int i = 0; i < k; ++i) out_fetch[(size_t)t * k + i] = i < nf ? fetch[i] : -1;
      if (out_nfetch) out_nfetch[t] = nf;
      if (out_resident) {
        int* r = out_resident + (size_t)t * C;
        int nr = 0;
        for (int c = 0; c < C; ++c) if (slot_block[c] >= 0) r[nr++] = slot_block[c];
        qsort(r, (size_t)nr, sizeof(int), orc_int_cmp);
        for (int c = nr; c < C; ++c) r[c] = -1;
      }
    } else {
      if (out_fetch) for (int i = 0; i < k; ++i) out_fetch[(size_t)t * k + i] = -1;
      if (out_nfetch) out_nfetch[t] = 0;
    }

    if (out_o && attend_mask && attend_mask[t]) {
      int nr = 0;
      for (int i = 0; i < ns; ++i)
        for (int j = 0; j < P; ++j) rows[nr++] = sel[i] * P + j;
      for (int j = 0; j < tail; ++j) rows[nr++] = n * P + j;
      orc_attend(q + (size_t)t * G * d, G, d, K, V, rows, nr, out_o + (size_t)t * G * d);
    }

    memcpy(prev, sel, sizeof(int) * (size_t)ns);
    n_prev = ns;

    if (cfg->append && tail == P) {
      orc_pool_keys(K + (size_t)n * P * d, R, Q, d, kbar + (size_t)n * R * d);
      n += 1;
      tail = 0;
    }
  }

  free(kbar); free(score); free(ge); free(ge_new); free(prev); free(sel);
  free(slot_block); free(last_used); free(fetch); free(fetch_slot); free(rows); free(forced);
  return rc;
}

/* Many independent units, in parallel over units when built with OpenMP.  The
 * arrays are the per-unit arrays of orc_run_unit stacked along a leading unit
 * axis.  Returns the number of threads used (negative on error). */
int orc_run_units(const orc_cfg* cfg, int n_units, const uint16_t* K, const uint16_t* V,
                  const float* a, const uint16_t* q, const unsigned char* attend_mask,
                  int* out_sel, int* out_nfetch, double* out_o) {
  const size_t kv = (size_t)cfg->max_blocks * cfg->P * cfg->d;
  const size_t qs = (size_t)cfg->steps * cfg->G * cfg->d;
  const int k = cfg->k_q + cfg->k_e;
  int bad = 0, threads = 1;
#ifdef _OPENMP
#pragma omp parallel
  {
#pragma omp single
    threads = omp_get_num_threads();
  }
#pragma omp parallel for schedule(dynamic, 1) reduction(|: bad)
#endif
  for (int u = 0; u < n_units; ++u) {
    int rc = orc_run_unit(cfg, K + u * kv, V + u * kv, a + (size_t)u * cfg->max_blocks,
                          q + u * qs, attend_mask,
                          out_sel ? out_sel + (size_t)u * cfg->steps * k : NULL, NULL, NULL,
                          out_nfetch ? out_nfetch + (size_t)u * cfg->steps : NULL, NULL,
                          out_o ? out_o + u * qs : NULL, NULL, NULL);
    if (rc != 0) bad |= 1;
  }
  return bad ? -1 : threads;
}
