/*
 * HiLS attention forward: CPU oracle.  TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously-correct definition that the CUDA
 * path is checked against.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load it; the product path never calls it.  It shares
 * no code with the CUDA library: it has its own storage readers, its own
 * cache addressing and its own selection.  All arithmetic is float64 on
 * inputs that are already rounded to their storage type (float32 or bf16).
 *
 * The method (HiLS, "Hierarchical Sparse Attention Done Right"):
 *   - the sequence is cut into fixed chunks of S tokens, each summarised by a
 *     landmark key (ai-feeds.com digest, section "输入与分块");
 *   - a low-rank query calibration q~ = q + (qA)B feeds retrieval only
 *     (same section; the oopus.info review, section 二, "低秩投影");
 *   - the calibrated query scores every causally visible chunk's landmark
 *     and the top-k chunks are retrieved (digest, "关键模块" items 1 and 2;
 *     review, section 二 first step);
 *   - the query attends to each retrieved chunk independently with an
 *     ordinary softmax, giving one output per chunk (digest, "关键模块" item 2;
 *     chatpaper abstract: "each query performs attention independently with
 *     each retrieved chunk");
 *   - the chunk outputs are fused with weights from the retrieval scores
 *     (digest item 2; review, "融合"; abstract: "fused according to chunk
 *     retrieval scores"), the outer softmax of the digest's hierarchical
 *     softmax (item 1).
 *
 * Readings where the pages are silent (fixed here and in the design notes):
 *   - score scale 1/sqrt(d); scorer is the dot product with q~;
 *   - one landmark per chunk per KV head, supplied as an input, so the inner
 *     softmax over a chunk's landmarks is the identity;
 *   - the own chunk c(i) = floor(i/S) is always selected and counts toward k;
 *     the other k-1 slots are the best candidates j < c(i), ordered by
 *     (score descending, chunk index ascending);
 *   - the own chunk's weight uses its landmark score like any other chunk;
 *   - fewer candidates than k-1: all are taken, idx pads with -1, w with 0;
 *   - the per-chunk attention uses the raw q (calibration serves retrieval),
 *     scale 1/sqrt(d), keys restricted to positions <= i in the own chunk;
 *   - A [d][r] and B [r][d] are shared by all heads; GQA query head h reads
 *     KV head h / (Hq/Hkv) and scores that head's landmarks;
 *   - fusion weights w = softmax of the selected chunks' scores.
 *
 * Storage (same conventions as the library, written out independently):
 *   landmarks[b][j][g][e]                    (batch, chunk, kv head, element)
 *   pages[p][kind][g][s][e]                  kind 0 = K, 1 = V, s = slot in chunk
 *   block_table[b][j] = physical page of logical chunk j of sequence b
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int32_t batch, n_q_heads, n_kv_heads, head_dim, chunk_size, top_k, calib_rank, dtype;
} ocfg;  /* dtype: 0 = float32, 1 = bf16 (storage of q, K, V, landmarks) */

/* ---- storage readers ---------------------------------------------------- */
static double ld(const void* p, int dtype, int64_t i) {
  if (dtype == 0) return (double)((const float*)p)[i];
  uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static int64_t kv_index(const ocfg* c, const int32_t* block_table, int32_t max_chunks, int b,
                        int64_t t, int kind, int g, int e) {
  int64_t j = t / c->chunk_size;
  int64_t page = block_table[(int64_t)b * max_chunks + j];
  int64_t s = t % c->chunk_size;
  return (((page * 2 + kind) * c->n_kv_heads + g) * c->chunk_size + s) * c->head_dim + e;
}

/* ---- a1: calibration q~ = q + (q A) B ----------------------------------- */
void oracle_calibrate(const double* q, const float* A, const float* B, int d, int r,
                      double* qt) {
  double* t = (double*)malloc(sizeof(double) * (r > 0 ? r : 1));
  for (int a = 0; a < r; ++a) {
    double acc = 0.0;
    for (int e = 0; e < d; ++e) acc += q[e] * (double)A[(int64_t)e * r + a];
    t[a] = acc;
  }
  for (int e = 0; e < d; ++e) {
    double acc = 0.0;
    for (int a = 0; a < r; ++a) acc += t[a] * (double)B[(int64_t)a * d + e];
    qt[e] = q[e] + acc;
  }
  free(t);
}

/* ---- a2: landmark score s_j = q~ . lm[b][j][g] / sqrt(d) ---------------- */
static double landmark_score(const ocfg* c, const double* qt, const void* landmarks,
                             int32_t max_chunks, int b, int g, int64_t j) {
  const int d = c->head_dim;
  int64_t base = (((int64_t)b * max_chunks + j) * c->n_kv_heads + g) * d;
  double acc = 0.0;
  for (int e = 0; e < d; ++e) acc += qt[e] * ld(landmarks, c->dtype, base + e);
  return acc / sqrt((double)d);
}

/* ---- a3: selection ------------------------------------------------------
 * Slot 0 is the own chunk.  Slots 1..k-1 take the best remaining candidate
 * j < own, one at a time: the largest score, and among equal scores the
 * smallest j (strict '>' while scanning j upward keeps the first).  Returns
 * the number of selected chunks; *gap is the score margin between the last
 * chosen candidate and the best candidate left out (+inf if none is left).
 */
static int select_chunks(const double* s, int64_t own, int k, int32_t* idx, double* gap) {
  int n = 1;
  idx[0] = (int32_t)own;
  char* taken = (char*)calloc((size_t)(own > 0 ? own : 1), 1);
  double last = INFINITY;
  for (int slot = 1; slot < k && slot <= own; ++slot) {
    int64_t best = -1;
    for (int64_t j = 0; j < own; ++j) {
      if (taken[j]) continue;
      if (best < 0 || s[j] > s[best]) best = j;
    }
    taken[best] = 1;
    idx[n++] = (int32_t)best;
    last = s[best];
  }
  for (int slot = n; slot < k; ++slot) idx[slot] = -1;
  if (gap) {
    double best_left = -INFINITY;
    for (int64_t j = 0; j < own; ++j)
      if (!taken[j] && s[j] > best_left) best_left = s[j];
    *gap = (best_left == -INFINITY) ? INFINITY : (n > 1 ? last - best_left : INFINITY);
  }
  free(taken);
  return n;
}

/* ---- a4: fusion weights w = softmax(selected scores) -------------------- */
static void fusion_weights(const double* ssel, int n, int k, double* w) {
  double m = -INFINITY;
  for (int a = 0; a < n; ++a) m = ssel[a] > m ? ssel[a] : m;
  double z = 0.0;
  for (int a = 0; a < n; ++a) z += exp(ssel[a] - m);
  for (int a = 0; a < n; ++a) w[a] = exp(ssel[a] - m) / z;
  for (int a = n; a < k; ++a) w[a] = 0.0;
}

/* ---- a5: independent softmax attention of raw q over one chunk --------- */
static void chunk_attention(const ocfg* c, const double* q, const void* pages,
                            const int32_t* block_table, int32_t max_chunks, int b, int g,
                            int64_t j, int64_t pos, double* o /* [d] */) {
  const int d = c->head_dim, S = c->chunk_size;
  int64_t t0 = j * S;
  int64_t t1 = t0 + S - 1;
  if (t1 > pos) t1 = pos; /* own chunk: keys at positions <= pos only */
  int64_t nk = t1 - t0 + 1;
  double* logit = (double*)malloc(sizeof(double) * (size_t)nk);
  double m = -INFINITY;
  for (int64_t t = t0; t <= t1; ++t) {
    double acc = 0.0;
    for (int e = 0; e < d; ++e)
      acc += q[e] * ld(pages, c->dtype, kv_index(c, block_table, max_chunks, b, t, 0, g, e));
    logit[t - t0] = acc / sqrt((double)d);
    if (logit[t - t0] > m) m = logit[t - t0];
  }
  double z = 0.0;
  for (int64_t a = 0; a < nk; ++a) z += exp(logit[a] - m);
  for (int e = 0; e < d; ++e) o[e] = 0.0;
  for (int64_t t = t0; t <= t1; ++t) {
    double p = exp(logit[t - t0] - m) / z;
    for (int e = 0; e < d; ++e)
      o[e] += p * ld(pages, c->dtype, kv_index(c, block_table, max_chunks, b, t, 1, g, e));
  }
  free(logit);
}

static int kv_head_of(const ocfg* c, int h) { return h / (c->n_q_heads / c->n_kv_heads); }

/* ---- one query row: a1..a6 ---------------------------------------------- */
static void hils_row(const ocfg* c, const double* q, int b, int h, int64_t pos, const float* A,
                     const float* B, const void* pages, const int32_t* block_table,
                     int32_t max_chunks, const void* landmarks, const int32_t* forced,
                     double* out, int32_t* idx, double* w, double* ssel_out, double* gap) {
  const int d = c->head_dim, k = c->top_k, g = kv_head_of(c, h);
  const int64_t own = pos / c->chunk_size;
  double* qt = (double*)malloc(sizeof(double) * d);
  oracle_calibrate(q, A, B, d, c->calib_rank, qt);

  double* ssel = (double*)malloc(sizeof(double) * k);
  int n;
  if (forced) {
    n = 0;
    for (int a = 0; a < k; ++a) {
      idx[a] = forced[a];
      if (forced[a] >= 0) ++n;
    }
    for (int a = 0; a < n; ++a)
      ssel[a] = landmark_score(c, qt, landmarks, max_chunks, b, g, idx[a]);
    if (gap) *gap = NAN;
  } else {
    double* s = (double*)malloc(sizeof(double) * (size_t)(own + 1));
    for (int64_t j = 0; j <= own; ++j) s[j] = landmark_score(c, qt, landmarks, max_chunks, b, g, j);
    n = select_chunks(s, own, k, idx, gap);
    for (int a = 0; a < n; ++a) ssel[a] = s[idx[a]];
    free(s);
  }
  fusion_weights(ssel, n, k, w);
  if (ssel_out) {
    for (int a = 0; a < k; ++a) ssel_out[a] = a < n ? ssel[a] : -INFINITY;
  }

  if (out) {
    double* o = (double*)malloc(sizeof(double) * d);
    for (int e = 0; e < d; ++e) out[e] = 0.0;
    for (int a = 0; a < n; ++a) {
      chunk_attention(c, q, pages, block_table, max_chunks, b, g, idx[a], pos, o);
      for (int e = 0; e < d; ++e) out[e] += w[a] * o[e];
    }
    free(o);
  }
  free(ssel);
  free(qt);
}

/* ---- exported entry points --------------------------------------------- */

/* Rows are given explicitly: q_rows[n][d] in storage dtype, with each row's
 * sequence b, query head h and absolute position pos.  pages may be NULL
 * (selection and weights only; out is then not written).  forced_idx, when
 * given, replaces the selection by the listed chunks ([n][k], -1 pads,
 * slot 0 must be the own chunk).  Returns 0, or -1 on a bad argument. */
int oracle_hils_rows(const ocfg* c, int64_t n_rows, const void* q_rows, const int32_t* row_b,
                     const int32_t* row_h, const int64_t* row_pos, const float* A, const float* B,
                     const void* pages, const int32_t* block_table, int32_t max_chunks,
                     const void* landmarks, const int32_t* forced_idx, double* out,
                     int32_t* idx, double* w, double* sel_scores, double* gap) {
  if (!c || c->head_dim <= 0 || c->chunk_size <= 0 || c->top_k <= 0 || c->n_kv_heads <= 0 ||
      c->n_q_heads % c->n_kv_heads != 0)
    return -1;
  const int d = c->head_dim, k = c->top_k;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < n_rows; ++r) {
    double* q = (double*)malloc(sizeof(double) * d);
    for (int e = 0; e < d; ++e) q[e] = ld(q_rows, c->dtype, r * d + e);
    hils_row(c, q, row_b[r], row_h[r], row_pos[r], A, B, pages, block_table, max_chunks,
             landmarks, forced_idx ? forced_idx + r * k : NULL, (pages && out) ? out + r * d : NULL,
             idx + r * k, w + r * k, sel_scores ? sel_scores + r * k : NULL,
             gap ? gap + r : NULL);
    free(q);
  }
  return 0;
}

/* All landmark scores of the given rows: scores[n][n_cols], column j holds
 * s_j for j <= floor(pos/S) and -inf after it. */
int oracle_scores_rows(const ocfg* c, int64_t n_rows, const void* q_rows, const int32_t* row_b,
                       const int32_t* row_h, const int64_t* row_pos, const float* A,
                       const float* B, const void* landmarks, int32_t max_chunks, int32_t n_cols,
                       double* scores) {
  if (!c || c->n_kv_heads <= 0 || c->n_q_heads % c->n_kv_heads != 0) return -1;
  const int d = c->head_dim;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < n_rows; ++r) {
    double* q = (double*)malloc(sizeof(double) * d);
    double* qt = (double*)malloc(sizeof(double) * d);
    for (int e = 0; e < d; ++e) q[e] = ld(q_rows, c->dtype, r * d + e);
    oracle_calibrate(q, A, B, d, c->calib_rank, qt);
    int64_t own = row_pos[r] / c->chunk_size;
    for (int64_t j = 0; j < n_cols; ++j)
      scores[r * n_cols + j] =
          j <= own ? landmark_score(c, qt, landmarks, max_chunks, row_b[r],
                                    kv_head_of(c, row_h[r]), j)
                   : -INFINITY;
    free(qt);
    free(q);
  }
  return 0;
}

/* Selection and weights from given scores (a3, a4 alone): scores[n][n_cols]
 * with the row's own chunk at column floor(pos/S). */
int oracle_topk_rows(int64_t n_rows, const double* scores, int32_t n_cols, const int64_t* row_pos,
                     int32_t chunk_size, int32_t k, int32_t* idx, double* w, double* gap) {
  if (k <= 0 || chunk_size <= 0) return -1;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < n_rows; ++r) {
    const double* s = scores + r * n_cols;
    int64_t own = row_pos[r] / chunk_size;
    if (own >= n_cols) own = n_cols - 1;
    int32_t* ix = idx + r * k;
    int n = select_chunks(s, own, k, ix, gap ? gap + r : NULL);
    double* ssel = (double*)malloc(sizeof(double) * k);
    for (int a = 0; a < n; ++a) ssel[a] = s[ix[a]];
    fusion_weights(ssel, n, k, w + r * k);
    free(ssel);
  }
  return 0;
}

int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}
