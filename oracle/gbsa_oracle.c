/*
 * gbsa_oracle.c -- plain fp64 CPU reference for block-sparse paged GQA
 * attention (forward, and the gradients of its output at the end).  TEST
 * INFRASTRUCTURE ONLY: the tests, the smoke check
 * and the benchmark's CPU-baseline leg may call it; the product path never
 * does.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes, for each requested (global token row tg, query head h):
 *
 *   b      = the sequence holding tg          (cu_seqlens_q prefix sums)
 *   t      = tg - cu_seqlens_q[b]             (token index inside b)
 *   qs, qu = storage and used query length of b; ku = seqused_kv[b]
 *   G      = N1 / N2, kvh = h / G             (grouped query heads)
 *   qb     = (Q blocks of the sequences before b) + t / block_x
 *   n      = sparse_count[kvh][qb] clamped to [0, top_k]
 *   pos    = t + (ku - qu)                    (query position; bottom-right
 *                                              aligned causal mask)
 *   keys   = for every list entry j < n with lb = sparse_idx[kvh][qb][j]
 *            inside [0, ceil(ku/128)): the positions p = 128*lb + r,
 *            r in [0,128), that satisfy p < ku, p <= pos,
 *            (win_left  < 0 or p >= pos - win_left),
 *            (win_right < 0 or p <= pos + win_right);
 *            position p is stored in physical page block_table[b][lb], row r
 *            (paged pool), or in row cu_seqlens_kv[b] + p of k and v (TND).
 *   s_p    = scale * sum_d q[tg][h][d] * k[page][r][kvh][d]
 *   out    = sum_p exp(s_p - m) v_p / sum_p exp(s_p - m),  m = max_p s_p
 *   lse    = m + ln(sum_p exp(s_p - m))
 *   no key, or t >= qu:  out = 0, lse = -inf
 *
 * Sources: GBSA article (cf-1.com/news/4865651), "Function / sparse attention
 * mechanism" (the formula, the block split along S, selection by
 * sparseBlockIdx / sparseBlockCount from the paged cache); "Constraints"
 * (Q blocks counted over storage lengths, seqused dual-length semantics,
 * GQA N1 % N2 == 0, page size = blockShapeY = 128, PA_BBND stride rule);
 * "Mask" (maskType 1 = built-in causal); "Return values" (lse shape).
 * FA blog (ai6s.net), "three steps": the tiled online softmax is exactly
 * equal to this two-pass softmax, which is why the reference uses the
 * plain definition.  Readings where the pages are silent (head grouping
 * kvh = h / G, bottom-right causal alignment, the window's inclusive bounds,
 * logical block indices, duplicate entries counted twice, out-of-range
 * entries ignored, empty rows -> 0 / -inf, natural-log lse) are listed in
 * the design notes.
 *
 * Inputs are raw 16-bit patterns (uint16) of bf16 (dtype 0) or IEEE 754
 * binary16 (dtype 1) values; each is widened exactly to fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_PAGE 128

typedef struct {
  int32_t B, T, N1, N2, D, block_x, total_q_blocks, top_k, max_pages_per_seq, num_pages;
  int64_t kv_page_stride;
  double scale;
  int32_t win_left, win_right;
  double (*widen)(uint16_t); /* bf16 or fp16 bits -> exact fp64 */
  const uint16_t *q, *k, *v;
  const int32_t *sparse_idx, *sparse_count;
  const int64_t* cu_seqlens_q;
  const int32_t *seqused_q, *seqused_kv, *block_table;
  const int64_t* cu_seqlens_kv; /* TND K/V: [B+1] row offsets; NULL for the paged pool */
  const int64_t* rows; /* pairs (tg, h) */
  int64_t n_rows;
  double *out, *lse;
  double* out_abs; /* optional: per row and d, sum_p w_p |v_p[d]| (rounding-error scale) */
  double* gap_abs; /* optional: per row and d, sum_p w_p (m - s_p) |v_p[d]|, m = max_p s_p */
  int64_t* q_block_base; /* [B]: Q blocks of the sequences before b */
  int failed;            /* set to a nonzero code by a worker on bad input */
} oracle_ctx;

/* bf16 is the upper half of an IEEE 754 binary32. */
static double widen_bf16(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* IEEE 754 binary16: sign, 5 exponent bits (bias 15), 10 fraction bits.
 * Exponent 0 holds zero and the subnormals f * 2^-24; 31 holds inf / NaN. */
static double widen_fp16(uint16_t bits) {
  const int sign = bits >> 15, e = (bits >> 10) & 0x1f, f = bits & 0x3ff;
  double mag;
  if (e == 0)
    mag = ldexp((double)f, -24);
  else if (e == 31)
    mag = f ? NAN : INFINITY;
  else
    mag = ldexp((double)(1024 + f), e - 25); /* (1 + f / 1024) * 2^(e - 15) */
  return sign ? -mag : mag;
}

/* The exact fp64 values of n 16-bit patterns (dtype 0 bf16, 1 fp16); lets
 * the tests pin the decoding on its own.  Returns nonzero for a bad dtype. */
int gbsa_oracle_widen(int32_t dtype, const uint16_t* bits, int64_t n, double* out) {
  if (dtype != 0 && dtype != 1) return 1;
  for (int64_t i = 0; i < n; i++) out[i] = dtype ? widen_fp16(bits[i]) : widen_bf16(bits[i]);
  return 0;
}

/* Largest b with cu_seqlens_q[b] <= tg (sequences may be empty). */
static int32_t find_sequence(const oracle_ctx* c, int64_t tg) {
  int32_t lo = 0, hi = c->B - 1;
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) / 2;
    if (c->cu_seqlens_q[mid] <= tg) lo = mid; else hi = mid - 1;
  }
  /* skip empty sequences that share the same start */
  while (lo + 1 < c->B && c->cu_seqlens_q[lo + 1] <= tg) lo++;
  return lo;
}

/* Computes one (tg, h) row; scratch holds room for top_k*128 keys.  When
 * n_keys / kv_head are given they get the number of visible keys (their
 * scores, pages and rows are in score, key_page, key_row) and the KV head. */
static int one_row(const oracle_ctx* c, int64_t tg, int32_t h, double* out, double* lse,
                   double* out_abs, double* gap_abs, double* score, int64_t* key_page,
                   int32_t* key_row, int64_t* n_keys, int32_t* kv_head) {
  const int32_t D = c->D;
  for (int32_t d = 0; d < D; d++) out[d] = 0.0;
  if (out_abs)
    for (int32_t d = 0; d < D; d++) out_abs[d] = 0.0;
  if (gap_abs)
    for (int32_t d = 0; d < D; d++) gap_abs[d] = 0.0;
  *lse = -INFINITY;
  if (n_keys) *n_keys = 0;
  if (tg < 0 || tg >= c->T || h < 0 || h >= c->N1) return 1;

  const int32_t b = find_sequence(c, tg);
  const int64_t t = tg - c->cu_seqlens_q[b];
  const int64_t qs = c->cu_seqlens_q[b + 1] - c->cu_seqlens_q[b];
  const int64_t qu = c->seqused_q ? (int64_t)c->seqused_q[b] : qs;
  const int64_t ku = c->seqused_kv[b];
  if (t >= qu) return 0; /* rows past seqused_q: out 0, lse -inf */

  const int32_t G = c->N1 / c->N2;
  const int32_t kvh = h / G;
  const int64_t qb = c->q_block_base[b] + t / c->block_x;
  if (qb < 0 || qb >= c->total_q_blocks) return 2;
  int64_t n = c->sparse_count[(int64_t)kvh * c->total_q_blocks + qb];
  if (n < 0) n = 0;
  if (n > c->top_k) n = c->top_k;

  const int64_t pos = t + (ku - qu);
  const int64_t blocks_in_seq = (ku + ORACLE_PAGE - 1) / ORACLE_PAGE;
  const int32_t* list = c->sparse_idx + ((int64_t)kvh * c->total_q_blocks + qb) * c->top_k;

  /* Gather the visible keys, entry by entry, row by row. */
  int64_t nk = 0;
  for (int64_t j = 0; j < n; j++) {
    const int64_t lb = list[j];
    if (lb < 0 || lb >= blocks_in_seq) continue; /* out-of-range entries add nothing */
    int64_t page = -1;
    if (!c->cu_seqlens_kv) {
      page = c->block_table[(int64_t)b * c->max_pages_per_seq + lb];
      if (page < 0 || page >= c->num_pages) return 3;
    }
    for (int32_t r = 0; r < ORACLE_PAGE; r++) {
      const int64_t p = lb * ORACLE_PAGE + r;
      if (p >= ku) continue;
      if (p > pos) continue;
      if (c->win_left >= 0 && p < pos - c->win_left) continue;
      if (c->win_right >= 0 && p > pos + c->win_right) continue;
      if (c->cu_seqlens_kv) {
        /* TND: the token row of position p; the "page" stride is one row */
        key_page[nk] = c->cu_seqlens_kv[b] + p;
        key_row[nk] = 0;
      } else {
        key_page[nk] = page;
        key_row[nk] = r;
      }
      nk++;
    }
  }
  if (n_keys) *n_keys = nk;
  if (kv_head) *kv_head = kvh;
  if (nk == 0) return 0;

  const uint16_t* qrow = c->q + (tg * c->N1 + h) * (int64_t)D;
  for (int64_t i = 0; i < nk; i++) {
    const uint16_t* krow =
        c->k + key_page[i] * c->kv_page_stride + ((int64_t)key_row[i] * c->N2 + kvh) * D;
    double dot = 0.0;
    for (int32_t d = 0; d < D; d++) dot += c->widen(qrow[d]) * c->widen(krow[d]);
    score[i] = c->scale * dot;
  }

  /* Two-pass softmax: the maximum first, then the normalised weights. */
  double m = -INFINITY;
  for (int64_t i = 0; i < nk; i++) if (score[i] > m) m = score[i];
  double l = 0.0;
  for (int64_t i = 0; i < nk; i++) l += exp(score[i] - m);
  for (int64_t i = 0; i < nk; i++) {
    const double w = exp(score[i] - m) / l;
    const uint16_t* vrow =
        c->v + key_page[i] * c->kv_page_stride + ((int64_t)key_row[i] * c->N2 + kvh) * D;
    for (int32_t d = 0; d < D; d++) out[d] += w * c->widen(vrow[d]);
    if (out_abs)
      for (int32_t d = 0; d < D; d++) out_abs[d] += w * fabs(c->widen(vrow[d]));
    if (gap_abs)
      for (int32_t d = 0; d < D; d++) gap_abs[d] += w * (m - score[i]) * fabs(c->widen(vrow[d]));
  }
  *lse = m + log(l);
  return 0;
}

/* c->q_block_base[b] = Q blocks of the sequences before b, counted over
 * storage lengths ("Constraints: block split"); checks the prefix sums.
 * Allocates the array (the caller frees it) and returns 0, or an error code
 * with nothing allocated. */
static int q_block_bases(oracle_ctx* c) {
  c->q_block_base = (int64_t*)malloc(sizeof(int64_t) * (size_t)c->B);
  if (!c->q_block_base) return 11;
  const int64_t block_x = c->block_x;
  int64_t acc = 0;
  for (int32_t b = 0; b < c->B; b++) {
    c->q_block_base[b] = acc;
    const int64_t qs = c->cu_seqlens_q[b + 1] - c->cu_seqlens_q[b];
    if (qs < 0) { free(c->q_block_base); return 12; }
    acc += (qs + block_x - 1) / block_x;
  }
  if (acc != c->total_q_blocks || c->cu_seqlens_q[0] != 0 || c->cu_seqlens_q[c->B] != c->T) {
    free(c->q_block_base);
    return 13;
  }
  return 0;
}

typedef struct {
  oracle_ctx* c;
  int64_t begin, end;
} oracle_job;

static void* run_job(void* arg) {
  oracle_job* job = (oracle_job*)arg;
  oracle_ctx* c = job->c;
  const int64_t cap = (int64_t)c->top_k * ORACLE_PAGE;
  double* score = (double*)malloc(sizeof(double) * (size_t)cap);
  int64_t* key_page = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap);
  int32_t* key_row = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  if (!score || !key_page || !key_row) {
    c->failed = 4;
  } else {
    for (int64_t i = job->begin; i < job->end; i++) {
      const int rc = one_row(c, c->rows[2 * i], (int32_t)c->rows[2 * i + 1], c->out + i * c->D,
                             c->lse + i, c->out_abs ? c->out_abs + i * c->D : NULL,
                             c->gap_abs ? c->gap_abs + i * c->D : NULL, score, key_page, key_row,
                             NULL, NULL);
      if (rc) c->failed = rc;
    }
  }
  free(score);
  free(key_page);
  free(key_row);
  return NULL;
}

/*
 * Reference attention for n_rows (token, head) pairs given in `rows`
 * ([n_rows][2] int64: global token index, query head).  Writes out
 * [n_rows][D] and lse [n_rows] in fp64.  kv_page_stride is in elements.
 * seqused_q may be NULL (every storage token used).  dtype: 0 = bf16,
 * 1 = fp16 element bits in q, k, v.  cu_seqlens_kv == NULL: k and v are the
 * paged pool read through block_table; otherwise they are TND [T_kv][N2][D]
 * with sequence b in rows [cu_seqlens_kv[b], cu_seqlens_kv[b+1]) (block_table,
 * num_pages, max_pages_per_seq and kv_page_stride are then unused).  out_abs
 * (optional, [n_rows][D]) gets sum_p w_p |v_p[d]|, the scale of the error a
 * rounding of the weights can cause; gap_abs (optional, [n_rows][D]) gets
 * sum_p w_p (m - s_p) |v_p[d]| with m the row's largest score, the scale of
 * the error of weights whose exponent is rounded in proportion to its size
 * (s_p - m, up to a constant).  Returns 0 on success, nonzero if an
 * argument or a device-style value is outside its range.
 */
int gbsa_oracle_attention_rows(int32_t B, int32_t T, int32_t N1, int32_t N2, int32_t D,
                               int32_t block_x, int32_t total_q_blocks, int32_t top_k,
                               int32_t max_pages_per_seq, int32_t num_pages,
                               int64_t kv_page_stride, double scale, int32_t win_left,
                               int32_t win_right, int32_t dtype, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const int32_t* sparse_idx,
                               const int32_t* sparse_count, const int64_t* cu_seqlens_q,
                               const int32_t* seqused_q, const int32_t* seqused_kv,
                               const int32_t* block_table, const int64_t* cu_seqlens_kv,
                               const int64_t* rows, int64_t n_rows,
                               double* out, double* lse, double* out_abs, double* gap_abs,
                               int32_t n_threads) {
  if (B < 1 || T < 1 || N2 < 1 || N1 < N2 || N1 % N2 || D < 1 || block_x < 1 || top_k < 1 ||
      total_q_blocks < 1 || n_rows < 0 || (dtype != 0 && dtype != 1))
    return 10;
  if (!cu_seqlens_kv && (max_pages_per_seq < 1 || num_pages < 1)) return 10;
  if (cu_seqlens_kv) {
    /* TND rows: every sequence's used keys lie inside its own rows */
    if (cu_seqlens_kv[0] != 0) return 14;
    for (int32_t b = 0; b < B; b++)
      if (seqused_kv[b] < 0 || seqused_kv[b] > cu_seqlens_kv[b + 1] - cu_seqlens_kv[b]) return 14;
    kv_page_stride = (int64_t)N2 * D;
  }
  oracle_ctx c;
  memset(&c, 0, sizeof c);
  c.B = B; c.T = T; c.N1 = N1; c.N2 = N2; c.D = D; c.block_x = block_x;
  c.total_q_blocks = total_q_blocks; c.top_k = top_k;
  c.max_pages_per_seq = max_pages_per_seq; c.num_pages = num_pages;
  c.kv_page_stride = kv_page_stride; c.scale = scale;
  c.win_left = win_left; c.win_right = win_right;
  c.widen = dtype ? widen_fp16 : widen_bf16;
  c.q = q; c.k = k; c.v = v; c.sparse_idx = sparse_idx; c.sparse_count = sparse_count;
  c.cu_seqlens_q = cu_seqlens_q; c.seqused_q = seqused_q; c.seqused_kv = seqused_kv;
  c.block_table = block_table; c.cu_seqlens_kv = cu_seqlens_kv; c.rows = rows; c.n_rows = n_rows; c.out = out; c.lse = lse;
  c.out_abs = out_abs;
  c.gap_abs = gap_abs;

  const int qrc = q_block_bases(&c);
  if (qrc) return qrc;

  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  if (n_rows < n_threads) n_threads = n_rows > 0 ? (int32_t)n_rows : 1;
  pthread_t tid[256];
  oracle_job jobs[256];
  for (int32_t i = 0; i < n_threads; i++) {
    jobs[i].c = &c;
    jobs[i].begin = n_rows * i / n_threads;
    jobs[i].end = n_rows * (i + 1) / n_threads;
  }
  for (int32_t i = 1; i < n_threads; i++) pthread_create(&tid[i], NULL, run_job, &jobs[i]);
  run_job(&jobs[0]);
  for (int32_t i = 1; i < n_threads; i++) pthread_join(tid[i], NULL);
  free(c.q_block_base);
  return c.failed;
}

/*
 * Gradients of the attention output (training).  The GBSA article's
 * overview says the operator serves inference and training but gives no
 * backward; this is the gradient of the function computed above, taken
 * analytically and written out plainly.  For a row (tg, h) with visible
 * keys p (the same enumeration as one_row), weights w_p = exp(s_p - lse),
 * output O = sum_p w_p v_p and incoming gradient g = dout[tg][h]:
 *
 *   dv_p   += w_p g                                (dO / dv_p)
 *   dlt     = sum_d g[d] O[d]
 *   ds_p    = w_p (g . v_p - dlt)                  (softmax Jacobian)
 *   dq     += scale sum_p ds_p k_p
 *   dk_p   += scale ds_p q
 *
 * Rows with no key or past seqused_q contribute nothing.  dq is
 * [T][N1][D]; dk and dv have the layout of k and v (the paged pool
 * [num_pages][128][N2][D] with kv_page_stride, or TND [T_kv][N2][D]) and
 * are accumulated over every row and list entry that reads a key (a block
 * listed twice counts twice, as in the forward).  The *_abs outputs
 * (optional) get the same sums with every term replaced by its absolute
 * value, the term g.O of ds by sum_d |g[d]| sum_p w_p |v_p[d]|: the scale of
 * the rounding error of any evaluation order that forms the delta from a
 * computed O.
 * Single-threaded.  Returns 0 on success.
 */
int gbsa_oracle_attention_backward(int32_t B, int32_t T, int32_t N1, int32_t N2, int32_t D,
                                   int32_t block_x, int32_t total_q_blocks, int32_t top_k,
                                   int32_t max_pages_per_seq, int32_t num_pages,
                                   int64_t kv_page_stride, double scale, int32_t win_left,
                                   int32_t win_right, int32_t dtype, const uint16_t* q,
                                   const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                                   const int32_t* sparse_idx, const int32_t* sparse_count,
                                   const int64_t* cu_seqlens_q, const int32_t* seqused_q,
                                   const int32_t* seqused_kv, const int32_t* block_table,
                                   const int64_t* cu_seqlens_kv, double* dq, double* dk,
                                   double* dv, double* dq_abs, double* dk_abs, double* dv_abs) {
  if (B < 1 || T < 1 || N2 < 1 || N1 < N2 || N1 % N2 || D < 1 || block_x < 1 || top_k < 1 ||
      total_q_blocks < 1 || (dtype != 0 && dtype != 1))
    return 10;
  if (!cu_seqlens_kv && (max_pages_per_seq < 1 || num_pages < 1)) return 10;
  if (cu_seqlens_kv) {
    if (cu_seqlens_kv[0] != 0) return 14;
    for (int32_t b = 0; b < B; b++)
      if (seqused_kv[b] < 0 || seqused_kv[b] > cu_seqlens_kv[b + 1] - cu_seqlens_kv[b]) return 14;
    kv_page_stride = (int64_t)N2 * D;
  }
  oracle_ctx c;
  memset(&c, 0, sizeof c);
  c.B = B; c.T = T; c.N1 = N1; c.N2 = N2; c.D = D; c.block_x = block_x;
  c.total_q_blocks = total_q_blocks; c.top_k = top_k;
  c.max_pages_per_seq = max_pages_per_seq; c.num_pages = num_pages;
  c.kv_page_stride = kv_page_stride; c.scale = scale;
  c.win_left = win_left; c.win_right = win_right;
  c.widen = dtype ? widen_fp16 : widen_bf16;
  c.q = q; c.k = k; c.v = v; c.sparse_idx = sparse_idx; c.sparse_count = sparse_count;
  c.cu_seqlens_q = cu_seqlens_q; c.seqused_q = seqused_q; c.seqused_kv = seqused_kv;
  c.block_table = block_table; c.cu_seqlens_kv = cu_seqlens_kv;
  const int qrc = q_block_bases(&c);
  if (qrc) return qrc;
  const int64_t cap = (int64_t)top_k * ORACLE_PAGE;
  double* score = (double*)malloc(sizeof(double) * (size_t)cap);
  int64_t* key_page = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap);
  int32_t* key_row = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  double* out = (double*)malloc(sizeof(double) * (size_t)D);
  double* oabs = (double*)malloc(sizeof(double) * (size_t)D);
  int rc = (!score || !key_page || !key_row || !out || !oabs) ? 11 : 0;
  for (int64_t tg = 0; tg < T && !rc; tg++) {
    for (int32_t h = 0; h < N1 && !rc; h++) {
      double lse;
      int64_t nk = 0;
      int32_t kvh = 0;
      /* the visible keys of (tg, h) (pages, rows, scores), its KV head and O */
      rc = one_row(&c, tg, h, out, &lse, oabs, NULL, score, key_page, key_row, &nk, &kvh);
      if (rc || lse == -INFINITY) continue;
      const uint16_t* qrow = q + (tg * N1 + h) * (int64_t)D;
      const uint16_t* grow = dout + (tg * N1 + h) * (int64_t)D;
      /* dlt_abs scales the error of a delta formed from a computed O: every
         O[d] errs in proportion to sum_p w_p |v_p[d]| (oabs), not to |O[d]| */
      double dlt = 0.0, dlt_abs = 0.0;
      for (int32_t d = 0; d < D; d++) {
        dlt += c.widen(grow[d]) * out[d];
        dlt_abs += fabs(c.widen(grow[d])) * oabs[d];
      }
      double* dqr = dq + (tg * N1 + h) * (int64_t)D;
      double* dqa = dq_abs ? dq_abs + (tg * N1 + h) * (int64_t)D : NULL;
      for (int64_t i = 0; i < nk; i++) {
        const int64_t base = key_page[i] * kv_page_stride + ((int64_t)key_row[i] * N2 + kvh) * D;
        const uint16_t* krow = k + base;
        const uint16_t* vrow = v + base;
        const double w = exp(score[i] - lse);
        double gv = 0.0, gv_abs = 0.0;
        for (int32_t d = 0; d < D; d++) {
          gv += c.widen(grow[d]) * c.widen(vrow[d]);
          gv_abs += fabs(c.widen(grow[d]) * c.widen(vrow[d]));
        }
        const double ds = w * (gv - dlt);
        const double ds_abs = w * (gv_abs + dlt_abs);
        for (int32_t d = 0; d < D; d++) {
          const double g = c.widen(grow[d]);
          dv[base + d] += w * g;
          dqr[d] += scale * ds * c.widen(krow[d]);
          dk[base + d] += scale * ds * c.widen(qrow[d]);
          if (dv_abs) dv_abs[base + d] += w * fabs(g);
          if (dqa) dqa[d] += scale * ds_abs * fabs(c.widen(krow[d]));
          if (dk_abs) dk_abs[base + d] += scale * ds_abs * fabs(c.widen(qrow[d]));
        }
      }
    }
  }
  free(score); free(key_page); free(key_row); free(out); free(oabs);
  free(c.q_block_base);
  return rc;
}

