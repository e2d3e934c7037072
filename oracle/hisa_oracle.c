/*
 * CPU oracle for the HISA token-selection indexer and the flat DSA indexer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
 * CUDA library is checked against.  Only the test-suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it; the product path never does.
 * It shares no code, header or table with the CUDA library.
 *
 * Sources (all statements restated in our own words):
 *   [HISA]  aitrends.kr, "HISA: 세밀한 희소 어텐션을 위한 효율적인 계층적 인덱싱"
 *           (summary of the HISA paper):
 *             [HISA/pool]   paragraph on block partition and mean pooling
 *                           (L tokens form M contiguous blocks of B; a block's
 *                           representative is the sum of its keys over their count),
 *             [HISA/stage1] paragraph on stage 1 (query . representative dot
 *                           product, causal mask, keep the top-m blocks, the first
 *                           block and the last two blocks are always kept),
 *             [HISA/stage2] paragraph on stage 2 (original DSA scoring on the
 *                           tokens of the selected blocks only, emit the top-k
 *                           token indices for the sparse attention operator),
 *             [HISA/kv]     paragraph on maintaining representatives at KV-cache
 *                           update time and keeping the DSA output structure,
 *             [HISA/varlen] paragraph on forced blocks under varlen packing.
 *   [DSA]   idea.jsleekr.com, "긴 컨텍스트 LLM이 느려지는 이유와 희소 어텐션(sparse
 *           attention)으로 해결하는 방법", section "DSA: 딥시크의 희소 어텐션"
 *           (each query scores every earlier key with a light dot product and
 *           keeps the top few).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - "last two blocks" = the query's own block and the block before it, counted
 *     inside m; if at most m blocks are eligible all of them are selected.
 *   - with m < 3 the forced blocks are kept in the order own, previous, first.
 *   - ties: lower block index wins in stage 1, lower token index wins in stage 2;
 *     output rows are ordered by score descending, padded with -1.
 *   - token scoring is a single-head dot product q.k; positions are
 *     sequence-local; a partial block is divided by the count of keys present.
 *
 * Arithmetic: bf16 inputs are widened exactly to double and every sum is taken
 * in double, in dimension order 0..d-1.
 */

#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NONFINITE 2
#define ORC_ERR_ALLOC 3

/* Test hook: a non-zero code plants one deliberate mistake so that the test
 * suite can show its pins catch it.  Zero (the default) is the oracle. */
static int g_mutation = 0;

void oracle_set_mutation(int code) { g_mutation = code; }
int oracle_get_mutation(void) { return g_mutation; }

static double bf16_value(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ------------------------------------------------------------------------- */
/* query-row bookkeeping                                                      */

typedef struct {
  const int32_t *cu_q, *cu_k, *seqlens;
  int S;
} seq_layout;

static int seq_len(const seq_layout *L, int s) {
  return L->seqlens ? L->seqlens[s] : L->cu_k[s + 1] - L->cu_k[s];
}

/* Map a global query row to (sequence, sequence-local position). The queries
 * of a sequence are its last q_len positions. Returns 0 on success. */
static int locate_query(const seq_layout *L, int row, int *s_out, int *pos_out) {
  int lo = 0, hi = L->S - 1, s = -1;
  while (lo <= hi) { /* last s with cu_q[s] <= row */
    int mid = (lo + hi) / 2;
    if (L->cu_q[mid] <= row) { s = mid; lo = mid + 1; } else { hi = mid - 1; }
  }
  while (s >= 0 && s < L->S && L->cu_q[s + 1] <= row) s++; /* skip empty sequences */
  if (s < 0 || s >= L->S) return -1;
  int qlen = L->cu_q[s + 1] - L->cu_q[s];
  int len = seq_len(L, s);
  int pos = len - qlen + (row - L->cu_q[s]);
  if (pos < 0 || pos >= len) return -1;
  *s_out = s;
  *pos_out = pos;
  return 0;
}

/* ------------------------------------------------------------------------- */
/* [HISA/pool] mean pooling                                                   */

int oracle_pool(const uint16_t *k, const int32_t *cu_k, const int32_t *seqlens, int S, int d,
                int B, double *reps) {
  if (!k || !cu_k || !reps || S < 0 || d <= 0 || B <= 0) return ORC_ERR_ARG;
  for (int s = 0; s < S; s++) {
    int start = cu_k[s];
    int len = seqlens ? seqlens[s] : cu_k[s + 1] - cu_k[s];
    if (start % B != 0 || len < 0 || start + len > cu_k[s + 1]) return ORC_ERR_ARG;
    int nblk = (len + B - 1) / B;
    for (int b = 0; b < nblk; b++) {
      int first = start + b * B;
      int count = len - b * B < B ? len - b * B : B;
      double *rep = reps + (size_t)(first / B) * d;
      for (int c = 0; c < d; c++) {
        double sum = 0.0;
        for (int t = 0; t < count; t++) {
          double v = bf16_value(k[(size_t)(first + t) * d + c]);
          if (!isfinite(v)) return ORC_ERR_NONFINITE;
          sum += v;
        }
        /* mutation 1: divide by B instead of by the number of keys present */
        rep[c] = sum / (double)(g_mutation == 1 ? B : count);
      }
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* scores                                                                     */

static double dot_bf16_double(const uint16_t *a, const double *b, int d) {
  double acc = 0.0;
  for (int c = 0; c < d; c++) acc += bf16_value(a[c]) * b[c];
  return acc;
}

static double dot_bf16_bf16(const uint16_t *a, const uint16_t *b, int d) {
  int dd = (g_mutation == 6) ? d - 1 : d; /* mutation 6: drop the last dimension */
  double acc = 0.0;
  for (int c = 0; c < dd; c++) acc += bf16_value(a[c]) * bf16_value(b[c]);
  return acc;
}

/* ------------------------------------------------------------------------- */
/* ordering: score descending, ties to the lower index                        */

typedef struct {
  double score;
  int32_t idx;
} cand;

/* flip_ties != 0 plants the "ties to the higher index" mistake (mutations 3, 5) */
static int cand_order(const cand *a, const cand *b, int flip_ties) {
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  if (flip_ties) return (a->idx > b->idx) ? -1 : (a->idx < b->idx);
  return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

static int block_cmp(const void *pa, const void *pb) {
  return cand_order((const cand *)pa, (const cand *)pb, g_mutation == 3);
}

static int token_cmp(const void *pa, const void *pb) {
  return cand_order((const cand *)pa, (const cand *)pb, g_mutation == 5);
}

static int int_cmp(const void *pa, const void *pb) {
  int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
  return (a < b) ? -1 : (a > b);
}

/* ------------------------------------------------------------------------- */
/* [HISA/stage1] block selection for one query                                */

/* Selects the blocks of one query; writes them in ascending order to out[0..m),
 * padding with -1; returns the number selected or -1 on error. scores_out (if not
 * NULL) receives the score of each selected block, aligned with out. tmp must hold
 * nblk entries. */
static int select_blocks_one(const uint16_t *qrow, const double *rep_base, int d, int B, int m,
                             int pos, cand *tmp, int32_t *out, double *scores_out) {
  int own = pos / B;
  int eligible = own + 1; /* blocks 0..own: every block that is not wholly after the query */
  int take_all = (g_mutation == 9) ? (eligible <= m + 1) : (eligible <= m);
  int nsel = 0;
  int32_t sel[4096 + 8];
  if (m > 4096) return -1;
  if (take_all) {
    for (int b = 0; b < eligible; b++) sel[nsel++] = b;
  } else {
    /* forced blocks, in priority order own, previous, first */
    int forced[3], nf = 0;
    int cand_forced[3] = {own, own - 1, 0};
    for (int t = 0; t < 3 && nf < m; t++) {
      int b = cand_forced[t];
      if (g_mutation == 2 && t == 1) continue; /* mutation 2: previous block not forced */
      if (g_mutation == 8 && t == 2) continue; /* mutation 8: first block not forced */
      int dup = 0;
      for (int u = 0; u < nf; u++) dup |= (forced[u] == b);
      if (!dup && b >= 0) forced[nf++] = b;
    }
    for (int u = 0; u < nf; u++) sel[nsel++] = forced[u];
    /* every other eligible block competes for the remaining m - |F| slots */
    int nc = 0;
    for (int b = 0; b < eligible; b++) {
      int is_forced = 0;
      for (int u = 0; u < nf; u++) is_forced |= (forced[u] == b);
      if (is_forced) continue;
      double sc = dot_bf16_double(qrow, rep_base + (size_t)b * d, d);
      if (g_mutation == 7) sc = -sc; /* mutation 7: keep the lowest-scoring blocks */
      tmp[nc].score = sc;
      tmp[nc].idx = b;
      nc++;
    }
    qsort(tmp, (size_t)nc, sizeof(cand), block_cmp);
    int free_slots = m - nf;
    for (int t = 0; t < free_slots && t < nc; t++) sel[nsel++] = tmp[t].idx;
  }
  qsort(sel, (size_t)nsel, sizeof(int32_t), int_cmp);
  for (int t = 0; t < m; t++) out[t] = t < nsel ? sel[t] : -1;
  if (scores_out) {
    for (int t = 0; t < m; t++)
      scores_out[t] = t < nsel ? dot_bf16_double(qrow, rep_base + (size_t)sel[t] * d, d) : 0.0;
  }
  return nsel;
}

/* ------------------------------------------------------------------------- */
/* [HISA/stage2] and [DSA]: exact top-k over an explicit candidate list        */

static void topk_emit(cand *c, int nc, int topk, int32_t *out_idx, double *out_scores) {
  qsort(c, (size_t)nc, sizeof(cand), token_cmp);
  for (int t = 0; t < topk; t++) {
    out_idx[t] = t < nc ? c[t].idx : -1;
    if (out_scores) out_scores[t] = t < nc ? c[t].score : 0.0;
  }
}

/* Candidate j of a query at position pos is admitted when j <= pos (token causal
 * mask). Mutation 4 uses j < pos instead. */
static int causal_ok(int j, int pos) { return g_mutation == 4 ? (j < pos) : (j <= pos); }

/* ------------------------------------------------------------------------- */
/* threaded runner over query rows                                           */

enum job_kind { JOB_BLOCKS, JOB_BLOCK_SCORES, JOB_TOKENS, JOB_DSA };

typedef struct {
  int kind;
  const uint16_t *q, *k;
  const double *reps;
  const int32_t *blocks;
  int nb;
  seq_layout L;
  int d, B, m, topk, max_blocks;
  const int32_t *rows;
  int nrows;
  int32_t *out_i32;
  double *out_f64;
  double *out_f64b;
  int next_row; /* shared work counter */
  pthread_mutex_t mu;
  int err;
} job;

static int job_row(job *J, int t) { return J->rows ? J->rows[t] : t; }

static int run_row(job *J, int t, cand *tmp, size_t tmp_cap) {
  int row = job_row(J, t), s, pos;
  if (locate_query(&J->L, row, &s, &pos)) return ORC_ERR_ARG;
  const uint16_t *qrow = J->q + (size_t)row * J->d;
  for (int c = 0; c < J->d; c++)
    if (!isfinite(bf16_value(qrow[c]))) return ORC_ERR_NONFINITE;
  int kbase = J->L.cu_k[s];
  if (J->kind == JOB_BLOCKS) {
    const double *rb = J->reps + (size_t)(kbase / J->B) * J->d;
    if ((size_t)(pos / J->B + 1) > tmp_cap) return ORC_ERR_ALLOC;
    int n = select_blocks_one(qrow, rb, J->d, J->B, J->m, pos, tmp, J->out_i32 + (size_t)t * J->m,
                              J->out_f64 ? J->out_f64 + (size_t)t * J->m : NULL);
    return n < 0 ? ORC_ERR_ARG : ORC_OK;
  }
  if (J->kind == JOB_BLOCK_SCORES) {
    /* every block's score (NaN where the block is wholly after the query) */
    const double *rb = J->reps + (size_t)(kbase / J->B) * J->d;
    double *o = J->out_f64 + (size_t)t * J->max_blocks;
    for (int b = 0; b < J->max_blocks; b++)
      o[b] = (b <= pos / J->B) ? dot_bf16_double(qrow, rb + (size_t)b * J->d, J->d) : NAN;
    return ORC_OK;
  }
  int nc = 0;
  if (J->kind == JOB_TOKENS) {
    const int32_t *bl = J->blocks + (size_t)t * J->nb;
    for (int u = 0; u < J->nb; u++) {
      int b = bl[u];
      if (b < 0) continue;
      if (b > pos / J->B) return ORC_ERR_ARG; /* a block wholly after the query */
      for (int v = 0; v < u; v++)
        if (bl[v] == b) return ORC_ERR_ARG; /* duplicate block */
      for (int j = b * J->B; j < (b + 1) * J->B && j <= pos; j++) {
        if (!causal_ok(j, pos)) continue;
        if ((size_t)nc >= tmp_cap) return ORC_ERR_ALLOC;
        double sc = dot_bf16_bf16(qrow, J->k + (size_t)(kbase + j) * J->d, J->d);
        if (!isfinite(sc)) return ORC_ERR_NONFINITE;
        tmp[nc].score = sc;
        tmp[nc].idx = j;
        nc++;
      }
    }
  } else { /* JOB_DSA: every causal key */
    for (int j = 0; j <= pos; j++) {
      if (!causal_ok(j, pos)) continue;
      if ((size_t)nc >= tmp_cap) return ORC_ERR_ALLOC;
      double sc = dot_bf16_bf16(qrow, J->k + (size_t)(kbase + j) * J->d, J->d);
      if (!isfinite(sc)) return ORC_ERR_NONFINITE;
      tmp[nc].score = sc;
      tmp[nc].idx = j;
      nc++;
    }
  }
  topk_emit(tmp, nc, J->topk, J->out_i32 + (size_t)t * J->topk,
            J->out_f64 ? J->out_f64 + (size_t)t * J->topk : NULL);
  return ORC_OK;
}

static size_t job_tmp_cap(job *J) {
  int maxlen = 1;
  for (int s = 0; s < J->L.S; s++) {
    int l = seq_len(&J->L, s);
    if (l > maxlen) maxlen = l;
  }
  if (J->kind == JOB_TOKENS) {
    size_t c = (size_t)J->nb * J->B + 1;
    return c < (size_t)maxlen + 1 ? c : (size_t)maxlen + 1;
  }
  return (size_t)maxlen + 1;
}

static void *worker(void *arg) {
  job *J = (job *)arg;
  size_t cap = job_tmp_cap(J);
  cand *tmp = (cand *)malloc(cap * sizeof(cand));
  if (!tmp) {
    pthread_mutex_lock(&J->mu);
    J->err = ORC_ERR_ALLOC;
    pthread_mutex_unlock(&J->mu);
    return NULL;
  }
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int t = J->next_row;
    int stop = J->err != ORC_OK;
    J->next_row += 16;
    pthread_mutex_unlock(&J->mu);
    if (stop || t >= J->nrows) break;
    int end = t + 16 < J->nrows ? t + 16 : J->nrows;
    for (; t < end; t++) {
      int e = run_row(J, t, tmp, cap);
      if (e != ORC_OK) {
        pthread_mutex_lock(&J->mu);
        if (J->err == ORC_OK) J->err = e;
        pthread_mutex_unlock(&J->mu);
        break;
      }
    }
  }
  free(tmp);
  return NULL;
}

static int run_job(job *J, int nthreads) {
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  J->next_row = 0;
  J->err = ORC_OK;
  pthread_mutex_init(&J->mu, NULL);
  pthread_t th[256];
  int started = 0;
  for (int i = 0; i < nthreads; i++) {
    if (pthread_create(&th[i], NULL, worker, J) == 0) started++;
    else break;
  }
  if (started == 0) worker(J);
  for (int i = 0; i < started; i++) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&J->mu);
  return J->err;
}

static int check_layout(const int32_t *cu_q, const int32_t *cu_k, int S, int total_q) {
  if (!cu_q || !cu_k || S < 0) return ORC_ERR_ARG;
  if (cu_q[0] != 0 || cu_q[S] != total_q) return ORC_ERR_ARG;
  for (int s = 0; s < S; s++)
    if (cu_q[s + 1] < cu_q[s] || cu_k[s + 1] < cu_k[s]) return ORC_ERR_ARG;
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* public entry points (ctypes)                                               */

int oracle_block_select(const uint16_t *q, const double *reps, const int32_t *cu_q,
                        const int32_t *cu_k, const int32_t *seqlens, int S, int total_q, int d,
                        int B, int m, const int32_t *rows, int nrows, int32_t *out_blocks,
                        double *out_block_scores, int nthreads) {
  if (!q || !reps || !out_blocks || d <= 0 || B <= 0 || m < 1) return ORC_ERR_ARG;
  if (check_layout(cu_q, cu_k, S, total_q)) return ORC_ERR_ARG;
  job J = {0};
  J.kind = JOB_BLOCKS;
  J.q = q;
  J.reps = reps;
  J.L = (seq_layout){cu_q, cu_k, seqlens, S};
  J.d = d;
  J.B = B;
  J.m = m;
  J.rows = rows;
  J.nrows = rows ? nrows : total_q;
  J.out_i32 = out_blocks;
  J.out_f64 = out_block_scores;
  return run_job(&J, nthreads);
}

int oracle_block_scores(const uint16_t *q, const double *reps, const int32_t *cu_q,
                        const int32_t *cu_k, const int32_t *seqlens, int S, int total_q, int d,
                        int B, int max_blocks, const int32_t *rows, int nrows, double *out,
                        int nthreads) {
  if (!q || !reps || !out || d <= 0 || B <= 0 || max_blocks < 1) return ORC_ERR_ARG;
  if (check_layout(cu_q, cu_k, S, total_q)) return ORC_ERR_ARG;
  job J = {0};
  J.kind = JOB_BLOCK_SCORES;
  J.q = q;
  J.reps = reps;
  J.L = (seq_layout){cu_q, cu_k, seqlens, S};
  J.d = d;
  J.B = B;
  J.max_blocks = max_blocks;
  J.rows = rows;
  J.nrows = rows ? nrows : total_q;
  J.out_f64 = out;
  return run_job(&J, nthreads);
}

int oracle_token_select(const uint16_t *q, const uint16_t *k, const int32_t *blocks, int nb,
                        const int32_t *cu_q, const int32_t *cu_k, const int32_t *seqlens, int S,
                        int total_q, int d, int B, int topk, const int32_t *rows, int nrows,
                        int32_t *out_idx, double *out_scores, int nthreads) {
  if (!q || !k || !blocks || !out_idx || nb < 1 || d <= 0 || B <= 0 || topk < 1)
    return ORC_ERR_ARG;
  if (check_layout(cu_q, cu_k, S, total_q)) return ORC_ERR_ARG;
  job J = {0};
  J.kind = JOB_TOKENS;
  J.q = q;
  J.k = k;
  J.blocks = blocks;
  J.nb = nb;
  J.L = (seq_layout){cu_q, cu_k, seqlens, S};
  J.d = d;
  J.B = B;
  J.topk = topk;
  J.rows = rows;
  J.nrows = rows ? nrows : total_q;
  J.out_i32 = out_idx;
  J.out_f64 = out_scores;
  return run_job(&J, nthreads);
}

int oracle_dsa(const uint16_t *q, const uint16_t *k, const int32_t *cu_q, const int32_t *cu_k,
               const int32_t *seqlens, int S, int total_q, int d, int topk, const int32_t *rows,
               int nrows, int32_t *out_idx, double *out_scores, int nthreads) {
  if (!q || !k || !out_idx || d <= 0 || topk < 1) return ORC_ERR_ARG;
  if (check_layout(cu_q, cu_k, S, total_q)) return ORC_ERR_ARG;
  job J = {0};
  J.kind = JOB_DSA;
  J.q = q;
  J.k = k;
  J.L = (seq_layout){cu_q, cu_k, seqlens, S};
  J.d = d;
  J.B = 1;
  J.topk = topk;
  J.rows = rows;
  J.nrows = rows ? nrows : total_q;
  J.out_i32 = out_idx;
  J.out_f64 = out_scores;
  return run_job(&J, nthreads);
}

/* Whole HISA indexer: pool -> stage 1 -> stage 2. reps_out (optional, [rows_k/B, d])
 * receives the fp64 representatives; blocks_out (optional, [nrows, m]) the selected
 * blocks in ascending order. */
int oracle_hisa(const uint16_t *q, const uint16_t *k, const int32_t *cu_q, const int32_t *cu_k,
                const int32_t *seqlens, int S, int total_q, int d, int B, int m, int topk,
                const int32_t *rows, int nrows, int32_t *out_idx, double *out_scores,
                int32_t *blocks_out, double *reps_out, int nthreads) {
  if (!q || !k || !out_idx || d <= 0 || B <= 0 || m < 1 || topk < 1) return ORC_ERR_ARG;
  if (check_layout(cu_q, cu_k, S, total_q)) return ORC_ERR_ARG;
  size_t nrep = (size_t)((cu_k[S] + B - 1) / B);
  int nr = rows ? nrows : total_q;
  double *reps = reps_out ? reps_out : (double *)calloc(nrep * (size_t)d + 1, sizeof(double));
  int32_t *blk = blocks_out ? blocks_out : (int32_t *)malloc(((size_t)nr * m + 1) * sizeof(int32_t));
  if (!reps || !blk) {
    if (!reps_out) free(reps);
    if (!blocks_out) free(blk);
    return ORC_ERR_ALLOC;
  }
  if (reps_out) memset(reps_out, 0, nrep * (size_t)d * sizeof(double));
  int e = oracle_pool(k, cu_k, seqlens, S, d, B, reps);
  if (e == ORC_OK)
    e = oracle_block_select(q, reps, cu_q, cu_k, seqlens, S, total_q, d, B, m, rows, nrows, blk,
                            NULL, nthreads);
  if (e == ORC_OK) {
    /* the token stage sees only the selected blocks (rows re-indexed 0..nr-1) */
    e = oracle_token_select(q, k, blk, m, cu_q, cu_k, seqlens, S, total_q, d, B, topk, rows, nrows,
                            out_idx, out_scores, nthreads);
  }
  if (!reps_out) free(reps);
  if (!blocks_out) free(blk);
  return e;
}

/* ------------------------------------------------------------------------- */
/* The sparse attention step that consumes the selected indices.
 *
 * [HISA/kv]: the top-k token indices keep the DSA output structure and go to the
 * sparse attention operator; [DSA]: attention is then computed only over the
 * selected tokens.  The pages name that operator but do not write out its
 * arithmetic; the reading used here is the textbook scaled dot-product attention
 * restricted to the selected tokens, with the heads of a query sharing its
 * selection and one key row and one value row per token shared by every head:
 *   s_j      = scale * q[i][h] . kv_key[j]          for the entries j >= 0 of idx[i]
 *   w_j      = exp(s_j - max s) / sum exp(s - max s)
 *   o[i][h]  = sum_j w_j * kv_val[j],   lse[i][h] = log sum_j exp(s_j)
 * A row with no valid index gets o = 0 and lse = -inf.  Sums in double, in index
 * order for the weights and dimension order for the dot products. */

typedef struct {
  const uint16_t *q, *k, *v;
  const int32_t *idx, *cu_q, *cu_k;
  int S, total_q, H, dv, topk;
  double scale;
  double *out, *lse;
  int next, err;
  pthread_mutex_t mu;
} att_job;

static void att_row(att_job *J, int row, double *s) {
  int sq = 0;
  while (sq + 1 < J->S && J->cu_q[sq + 1] <= row) sq++;
  const int64_t kbase = J->cu_k[sq];
  const int32_t *ir = J->idx + (int64_t)row * J->topk;
  for (int h = 0; h < J->H; h++) {
    const uint16_t *qh = J->q + ((int64_t)row * J->H + h) * J->dv;
    double *o = J->out + ((int64_t)row * J->H + h) * J->dv;
    for (int d = 0; d < J->dv; d++) o[d] = 0.0;
    double mx = -INFINITY;
    int n = 0;
    for (int t = 0; t < J->topk; t++) {
      int j = ir[t];
      if (j < 0) {
        if (g_mutation != 10) {
          s[t] = -INFINITY;
          continue;
        }
        j = 0;  /* planted mistake: padding read as token 0 */
      }
      const uint16_t *kr = J->k + (kbase + j) * J->dv;
      double acc = 0.0;
      for (int d = 0; d < J->dv; d++) acc += bf16_value(qh[d]) * bf16_value(kr[d]);
      s[t] = (g_mutation == 11 ? 1.0 : J->scale) * acc;
      if (s[t] > mx) mx = s[t];
      n++;
    }
    if (n == 0) {
      if (J->lse) J->lse[(int64_t)row * J->H + h] = -INFINITY;
      continue;
    }
    double sum = 0.0;
    for (int t = 0; t < J->topk; t++)
      if (s[t] != -INFINITY) sum += exp(s[t] - mx);
    for (int t = 0; t < J->topk; t++) {
      if (s[t] == -INFINITY) continue;
      const int j = ir[t] >= 0 ? ir[t] : 0;
      const double w = g_mutation == 12 ? exp(s[t] - mx) : exp(s[t] - mx) / sum;
      const uint16_t *vr = (g_mutation == 13 ? J->k : J->v) + (kbase + j) * J->dv;
      for (int d = 0; d < J->dv; d++) o[d] += w * bf16_value(vr[d]);
    }
    if (J->lse) J->lse[(int64_t)row * J->H + h] = mx + log(sum);
  }
}

static void *att_worker(void *arg) {
  att_job *J = (att_job *)arg;
  double *s = (double *)malloc(sizeof(double) * (size_t)(J->topk > 0 ? J->topk : 1));
  if (!s) {
    pthread_mutex_lock(&J->mu);
    J->err = ORC_ERR_ALLOC;
    pthread_mutex_unlock(&J->mu);
    return NULL;
  }
  for (;;) {
    pthread_mutex_lock(&J->mu);
    const int row = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (row >= J->total_q) break;
    att_row(J, row, s);
  }
  free(s);
  return NULL;
}

int oracle_sparse_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int32_t *idx, const int32_t *cu_q, const int32_t *cu_k, int S,
                            int total_q, int H, int dv, int topk, double scale, double *out,
                            double *lse, int nthreads) {
  if (!q || !k || !v || !idx || !cu_q || !cu_k || !out || S < 1 || total_q < 0 || H < 1 ||
      dv < 1 || topk < 1)
    return ORC_ERR_ARG;
  if (cu_q[0] != 0 || cu_q[S] != total_q) return ORC_ERR_ARG;
  att_job J = {q, k, v, idx, cu_q, cu_k, S, total_q, H, dv, topk, scale, out, lse, 0, 0,
               PTHREAD_MUTEX_INITIALIZER};
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  int started = 0;
  for (int t = 0; t < nthreads; t++)
    if (pthread_create(&th[t], NULL, att_worker, &J) == 0) started++;
  if (started == 0) att_worker(&J);
  for (int t = 0; t < started; t++) pthread_join(th[t], NULL);
  return J.err;
}
