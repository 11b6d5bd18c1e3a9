/*
 * s4r_oracle.c -- fp64 CPU oracle for S4R compressed-KV decode.
 *
 * TEST INFRASTRUCTURE ONLY (see s4r_oracle.h).  Plain loops in float64, one
 * step per paper equation, no blocking, fusion or reordering beyond what the
 * definitions state.  OpenMP only splits independent outputs across threads;
 * every output is a sequential sum, so results do not depend on the thread
 * count.
 *
 * Method source: "S^4R: Selective Sampling, Subspaces, and Sparse
 * Reconstruction for Compressed Long-Context KV Caching" (arXiv 2608.00528),
 * review page.  Readings taken where the page is silent are marked READING.
 */
#include "s4r_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int s4r_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

int s4r_oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#endif
  return s4r_oracle_threads();
}

/* Eq. 3 ("What carries the argument"): every non-sink token state s is stored
 * as its coefficients c = s . B in the rank-r basis B (D' x r). */
void s4r_oracle_encode(const double *S, int64_t n, int32_t d, const double *B,
                       int32_t r, double *C) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    for (int32_t j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int32_t e = 0; e < d; ++e) acc += S[t * d + e] * B[(int64_t)e * r + j];
      C[t * r + j] = acc;
    }
  }
}

/* Eq. 16 ("What carries the argument", "Referee Report: Summary"): a selected
 * row is rebuilt from its coefficients as k_hat = c . B^T. */
void s4r_oracle_reconstruct(const double *C, int64_t n, int32_t r,
                            const double *B, int32_t d, double *out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    for (int32_t e = 0; e < d; ++e) {
      double acc = 0.0;
      for (int32_t j = 0; j < r; ++j) acc += C[t * r + j] * B[(int64_t)e * r + j];
      out[t * d + e] = acc;
    }
  }
}

static int check_problem(const s4r_oracle_problem *p) {
  if (!p || p->n_heads_q <= 0 || p->n_heads_kv <= 0 || p->head_dim <= 0) return -1;
  if (p->n_heads_q % p->n_heads_kv != 0) return -1;
  if (p->rank_k <= 0 || p->rank_v <= 0 || p->query_window <= 0) return -1;
  if (p->n_sink < 0 || p->local_window < 0 || p->top_k < 0 || p->n_coeff < 0) return -1;
  if (p->pool_kernel < 1 || (p->pool_kernel > 1 && p->pool_kernel % 2 == 0)) return -1;
  if (p->pool_mode != S4R_ORACLE_POOL_MAX && p->pool_mode != S4R_ORACLE_POOL_AVG) return -1;
  if (p->row_mode != S4R_ORACLE_ROWS_CONCAT && p->row_mode != S4R_ORACLE_ROWS_PER_HEAD) return -1;
  return 0;
}

/* Query coefficients C_Q, one row per scoring row ("Core claim": queries are
 * projected into the key subspace; the query window is the sliding window of
 * query coefficients of Eqs. 8-10).
 *
 * READING (row formation).  The key basis spans D' = H_kv * d_h, so a query
 * row must be a D'-vector.  In ROWS_CONCAT mode row (w, j), j < G, is the
 * concatenation over kv groups g of query head g*G + j at window slot w; this
 * gives W*G rows, the G*W*r scoring term of the Appendix B complexity.  In
 * ROWS_PER_HEAD mode row (w, h) projects head h alone with the d_h rows of the
 * key basis that belong to its kv group g = h / G. */
static int64_t query_rows(const s4r_oracle_problem *p, double *cq /* [rows][r_k] or NULL */) {
  const int32_t W = p->query_window, Hq = p->n_heads_q, Hkv = p->n_heads_kv;
  const int32_t dh = p->head_dim, G = Hq / Hkv, r = p->rank_k;
  const int64_t n_rows = (p->row_mode == S4R_ORACLE_ROWS_CONCAT) ? (int64_t)W * G : (int64_t)W * Hq;
  if (!cq) return n_rows;
  for (int64_t row = 0; row < n_rows; ++row) {
    for (int32_t k = 0; k < r; ++k) {
      double acc = 0.0;
      if (p->row_mode == S4R_ORACLE_ROWS_CONCAT) {
        const int32_t w = (int32_t)(row / G), j = (int32_t)(row % G);
        for (int32_t g = 0; g < Hkv; ++g)
          for (int32_t t = 0; t < dh; ++t) {
            const double qv = p->q[((int64_t)w * Hq + (g * G + j)) * dh + t];   /* Q'[w][j][g*dh + t] */
            acc += qv * p->basis_k[(int64_t)(g * dh + t) * r + k];
          }
      } else {
        const int32_t w = (int32_t)(row / Hq), h = (int32_t)(row % Hq), g = h / G;
        for (int32_t t = 0; t < dh; ++t)
          acc += p->q[((int64_t)w * Hq + h) * dh + t] * p->basis_k[(int64_t)(g * dh + t) * r + k];
      }
      cq[row * r + k] = acc;
    }
  }
  return n_rows;
}

/* Latent relevance scoring, Eqs. 8-10 ("major comment 2", §3.2.2):
 *   Z = C_Q . C_K^T / sqrt(r)   (the scale is the one Eq. 8 prints),
 *   softmax of each row of Z over all L_c cached coefficient rows,
 *   score[i] = sum over rows of the softmax probabilities.
 * READING: the softmax domain is every coefficient row (sinks hold no
 * coefficients); aggregation over heads and the query window is a plain sum. */
int s4r_oracle_scores(const s4r_oracle_problem *p, double *scores) {
  if (check_problem(p)) return -1;
  const int64_t L = p->n_coeff;
  const int32_t r = p->rank_k;
  if (L == 0) return 0;
  const int64_t n_rows = query_rows(p, NULL);
  double *cq = (double *)malloc(sizeof(double) * n_rows * r);
  double *z = (double *)malloc(sizeof(double) * n_rows * L);
  double *row_max = (double *)malloc(sizeof(double) * n_rows);
  double *row_sum = (double *)malloc(sizeof(double) * n_rows);
  if (!cq || !z || !row_max || !row_sum) { free(cq); free(z); free(row_max); free(row_sum); return -3; }
  query_rows(p, cq);
  const double inv_sqrt_r = 1.0 / sqrt((double)r);

  /* Eq. 8: latent logits. */
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < L; ++i)
    for (int64_t row = 0; row < n_rows; ++row) {
      double acc = 0.0;
      for (int32_t k = 0; k < r; ++k) acc += cq[row * r + k] * p->coeff_k[i * r + k];
      z[row * L + i] = acc * inv_sqrt_r;
    }
  /* Eq. 9: softmax statistics of each row. */
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < n_rows; ++row) {
    double m = -INFINITY;
    for (int64_t i = 0; i < L; ++i) m = fmax(m, z[row * L + i]);
    double s = 0.0;
    for (int64_t i = 0; i < L; ++i) s += exp(z[row * L + i] - m);
    row_max[row] = m;
    row_sum[row] = s;
  }
  /* Eq. 10: aggregate the probabilities of every row onto each position. */
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < L; ++i) {
    double acc = 0.0;
    for (int64_t row = 0; row < n_rows; ++row)
      acc += exp(z[row * L + i] - row_max[row]) / row_sum[row];
    scores[i] = acc;
  }
  free(cq); free(z); free(row_max); free(row_sum);
  return 0;
}

/* Score pooling with kernel kappa ("free parameters": pooling kernel 7, taken
 * from SnapKV; the referee report lists the pooling/aggregation choices as
 * open).  READING: stride 1, same padding, over the candidate positions only;
 * kappa must be odd.  The window of position i is j = i - kappa/2 ..
 * i + kappa/2; neighbours outside [0, n_cand) are left out, so
 *   POOL_MAX: pooled[i] = max of scores[j] over the in-range j,
 *   POOL_AVG: pooled[i] = (sum of scores[j] over the in-range j) / (their count). */
int s4r_oracle_pool(const double *scores, int64_t n_cand, int32_t pool_kernel, int32_t pool_mode,
                    double *pooled) {
  if (pool_kernel < 1 || pool_kernel % 2 == 0) return -1;
  if (pool_mode != S4R_ORACLE_POOL_MAX && pool_mode != S4R_ORACLE_POOL_AVG) return -1;
  const int64_t half = pool_kernel / 2;
  for (int64_t i = 0; i < n_cand; ++i) {
    double m = -INFINITY, sum = 0.0;
    int64_t count = 0;
    for (int64_t j = i - half; j <= i + half; ++j)
      if (j >= 0 && j < n_cand) {
        m = fmax(m, scores[j]);
        sum += scores[j];
        count += 1;
      }
    pooled[i] = (pool_mode == S4R_ORACLE_POOL_MAX) ? m : sum / (double)count;
  }
  return 0;
}

typedef struct { double v; int64_t i; } keyed;

/* Larger score first; equal scores: smaller position first. */
static int by_score_desc(const void *a, const void *b) {
  const keyed *x = (const keyed *)a, *y = (const keyed *)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int by_int_asc(const void *a, const void *b) {
  const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x > y) - (x < y);
}

static int64_t n_candidates(const s4r_oracle_problem *p) {
  const int64_t c = p->n_coeff - p->local_window;
  return c > 0 ? c : 0;
}

/* Selection, Eqs. 13-15: the local window is always kept, and the top-k
 * global positions are chosen among the rows before it ("Core claim":
 * only the local window plus top-k global positions are reconstructed).
 * READING: candidates are coefficient rows 0 .. L_c-w-1; equal scores go to
 * the lower position; fewer than k candidates -> all of them, -1 padding. */
int s4r_oracle_select(const s4r_oracle_problem *p, const double *scores, int32_t *idx) {
  if (check_problem(p)) return -1;
  const int64_t n_cand = n_candidates(p);
  const int32_t k = p->top_k;
  for (int32_t e = 0; e < k; ++e) idx[e] = -1;
  if (n_cand == 0 || k == 0) return 0;
  const double *rank_by = scores;
  double *pooled = NULL;
  if (p->pool_kernel > 1) {
    pooled = (double *)malloc(sizeof(double) * n_cand);
    if (!pooled) return -3;
    s4r_oracle_pool(scores, n_cand, p->pool_kernel, p->pool_mode, pooled);
    rank_by = pooled;
  }
  keyed *all = (keyed *)malloc(sizeof(keyed) * n_cand);
  if (!all) { free(pooled); return -3; }
  for (int64_t i = 0; i < n_cand; ++i) { all[i].v = rank_by[i]; all[i].i = i; }
  qsort(all, (size_t)n_cand, sizeof(keyed), by_score_desc);
  const int64_t n_take = n_cand < k ? n_cand : k;
  for (int64_t e = 0; e < n_take; ++e) idx[e] = (int32_t)(all[e].i + p->n_sink);
  qsort(idx, (size_t)n_take, sizeof(int32_t), by_int_asc);
  free(all);
  free(pooled);
  return 0;
}

/* Sparse reconstruction + exact attention, Eqs. 16-18 ("Core claim",
 * "assumptions": the first s tokens are attention sinks kept in full
 * precision).  The current query (window slot W-1) of head h attends over the
 * sinks and the rebuilt selected rows, restricted to the d_h-slice of its kv
 * group g = h / G.  READING: logits scale 1/sqrt(d_h), contiguous GQA groups,
 * rebuilt rows kept in float64 (never rounded to a storage type). */
int s4r_oracle_decode_given_idx(const s4r_oracle_problem *p, const int32_t *idx,
                                int64_t n_idx, double *out) {
  if (check_problem(p)) return -1;
  const int64_t L = p->n_coeff;
  const int32_t Hq = p->n_heads_q, Hkv = p->n_heads_kv, dh = p->head_dim, G = Hq / Hkv;
  const int32_t Dp = Hkv * dh, W = p->query_window, s = p->n_sink;
  char *mark = (char *)calloc((size_t)(L > 0 ? L : 1), 1);
  if (!mark) return -3;
  for (int64_t e = 0; e < n_idx; ++e) {
    if (idx[e] < 0) continue;
    const int64_t i = (int64_t)idx[e] - s;
    if (i < 0 || i >= L) { free(mark); return -2; }
    mark[i] = 1;
  }
  for (int64_t i = L - p->local_window; i < L; ++i)
    if (i >= 0) mark[i] = 1;
  int64_t n_sel = 0;
  for (int64_t i = 0; i < L; ++i) n_sel += mark[i];
  int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (n_sel > 0 ? n_sel : 1));
  double *ck = (double *)malloc(sizeof(double) * (n_sel > 0 ? n_sel : 1) * p->rank_k);
  double *cv = (double *)malloc(sizeof(double) * (n_sel > 0 ? n_sel : 1) * p->rank_v);
  double *kh = (double *)malloc(sizeof(double) * (n_sel > 0 ? n_sel : 1) * Dp);
  double *vh = (double *)malloc(sizeof(double) * (n_sel > 0 ? n_sel : 1) * Dp);
  double *logit = (double *)malloc(sizeof(double) * (n_sel + s > 0 ? n_sel + s : 1));
  if (!rows || !ck || !cv || !kh || !vh || !logit) {
    free(mark); free(rows); free(ck); free(cv); free(kh); free(vh); free(logit);
    return -3;
  }
  n_sel = 0;
  for (int64_t i = 0; i < L; ++i)
    if (mark[i]) rows[n_sel++] = i;
  for (int64_t e = 0; e < n_sel; ++e) {
    memcpy(ck + e * p->rank_k, p->coeff_k + rows[e] * p->rank_k, sizeof(double) * p->rank_k);
    memcpy(cv + e * p->rank_v, p->coeff_v + rows[e] * p->rank_v, sizeof(double) * p->rank_v);
  }
  /* Eq. 16: rebuild only the selected rows. */
  s4r_oracle_reconstruct(ck, n_sel, p->rank_k, p->basis_k, Dp, kh);
  s4r_oracle_reconstruct(cv, n_sel, p->rank_v, p->basis_v, Dp, vh);

  const double scale = 1.0 / sqrt((double)dh);
  for (int32_t h = 0; h < Hq; ++h) {
    const int32_t g = h / G;
    const double *q = p->q + ((int64_t)(W - 1) * Hq + h) * dh;
    const int64_t n_keys = s + n_sel;
    for (int64_t t = 0; t < n_keys; ++t) {
      const double *key = (t < s) ? p->sink_k + t * Dp + (int64_t)g * dh
                                  : kh + (t - s) * Dp + (int64_t)g * dh;
      double acc = 0.0;
      for (int32_t e = 0; e < dh; ++e) acc += q[e] * key[e];
      logit[t] = acc * scale;
    }
    double m = -INFINITY;
    for (int64_t t = 0; t < n_keys; ++t) m = fmax(m, logit[t]);
    double z = 0.0;
    for (int64_t t = 0; t < n_keys; ++t) z += exp(logit[t] - m);
    double *o = out + (int64_t)h * dh;
    for (int32_t e = 0; e < dh; ++e) o[e] = 0.0;
    for (int64_t t = 0; t < n_keys; ++t) {
      const double pw = exp(logit[t] - m) / z;
      const double *val = (t < s) ? p->sink_v + t * Dp + (int64_t)g * dh
                                  : vh + (t - s) * Dp + (int64_t)g * dh;
      for (int32_t e = 0; e < dh; ++e) o[e] += pw * val[e];
    }
  }
  free(mark); free(rows); free(ck); free(cv); free(kh); free(vh); free(logit);
  return 0;
}

/* One decode step in the order the review's summary gives: latent scoring
 * (Eqs. 8-10), selection (Eqs. 13-15), sparse reconstruction and exact
 * attention (Eqs. 16-18). */
int s4r_oracle_decode_step(const s4r_oracle_problem *p, double *out, int32_t *idx,
                           double *scores) {
  if (check_problem(p)) return -1;
  double *sc = scores;
  if (!sc) {
    sc = (double *)malloc(sizeof(double) * (p->n_coeff > 0 ? p->n_coeff : 1));
    if (!sc) return -3;
  }
  int rc = s4r_oracle_scores(p, sc);
  if (!rc) rc = s4r_oracle_select(p, sc, idx);
  if (!rc) rc = s4r_oracle_decode_given_idx(p, idx, p->top_k, out);
  if (!scores) free(sc);
  return rc;
}
