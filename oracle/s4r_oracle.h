/*
 * s4r_oracle.h -- fp64 CPU oracle for S4R compressed-KV decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This library is the plain, slow, obviously
 * correct statement of what the decode path computes.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load it; the product
 * path (libs4r) never links, loads or calls it, and the two share no code.
 *
 * Source of the method: "S^4R: Selective Sampling, Subspaces, and Sparse
 * Reconstruction for Compressed Long-Context KV Caching" (arXiv 2608.00528),
 * its review page on pith.science.  Citations below name the section of that
 * page ("What carries the argument", "Core claim", "Referee Report: Summary",
 * "major comment 2", "free parameters", "assumptions") and the paper equation
 * the page refers to.
 *
 * Conventions: every array is fp64, row-major and contiguous.
 *   D' = n_heads_kv * head_dim, G = n_heads_q / n_heads_kv,
 *   L_c = number of coefficient rows; coefficient row i is absolute token
 *   position n_sink + i (the first n_sink tokens are the uncompressed sinks).
 */
#ifndef S4R_ORACLE_H
#define S4R_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  S4R_ORACLE_POOL_MAX = 0,      /* pooled score = largest neighbour score */
  S4R_ORACLE_POOL_AVG = 1       /* pooled score = mean of the in-range neighbour scores */
};

enum {
  S4R_ORACLE_ROWS_CONCAT = 0,   /* W*G rows, heads of one GQA slot concatenated to D' */
  S4R_ORACLE_ROWS_PER_HEAD = 1  /* W*H_q rows, each head projected with its own slice */
};

typedef struct {
  int32_t n_heads_q, n_heads_kv, head_dim;
  int32_t rank_k, rank_v;
  int32_t n_sink, local_window, top_k, query_window, pool_kernel;
  int32_t row_mode;             /* S4R_ORACLE_ROWS_* */
  int32_t pool_mode;            /* S4R_ORACLE_POOL_* (used when pool_kernel > 1) */
  int64_t n_coeff;              /* L_c */
  const double *q;              /* [W][H_q][d_h]; row W-1 is the current query */
  const double *coeff_k;        /* [L_c][rank_k] */
  const double *coeff_v;        /* [L_c][rank_v] */
  const double *basis_k;        /* [D'][rank_k] */
  const double *basis_v;        /* [D'][rank_v] */
  const double *sink_k;         /* [n_sink][D'] */
  const double *sink_v;         /* [n_sink][D'] */
} s4r_oracle_problem;

/* C[n][r] = S[n][d] . B[d][r]  (Eq. 3). */
void s4r_oracle_encode(const double *S, int64_t n, int32_t d, const double *B,
                       int32_t r, double *C);

/* out[n][d] = C[n][r] . B[d][r]^T  (Eq. 16, rebuilding rows from coefficients). */
void s4r_oracle_reconstruct(const double *C, int64_t n, int32_t r,
                            const double *B, int32_t d, double *out);

/* Latent relevance score of every coefficient row (Eqs. 8-10); scores[L_c].
 * Returns 0, or -1 on invalid shapes. */
int s4r_oracle_scores(const s4r_oracle_problem *p, double *scores);

/* Pooling of candidate scores with an odd window pool_kernel (stride 1,
 * same padding, candidates only): the largest (POOL_MAX) or the mean
 * (POOL_AVG) of the neighbours that lie inside [0, n_cand); pooled[n_cand]. */
int s4r_oracle_pool(const double *scores, int64_t n_cand, int32_t pool_kernel,
                    int32_t pool_mode, double *pooled);

/* Top-k global positions (Eqs. 13-15): idx[top_k] = absolute positions,
 * ascending, -1 padded.  Ranking uses the pooled scores when pool_kernel > 1. */
int s4r_oracle_select(const s4r_oracle_problem *p, const double *scores,
                      int32_t *idx);

/* Exact attention of the current query over sinks + the given absolute
 * positions (-1 entries ignored) + the local window (Eqs. 16-18);
 * out[H_q][d_h]. */
int s4r_oracle_decode_given_idx(const s4r_oracle_problem *p, const int32_t *idx,
                                int64_t n_idx, double *out);

/* One whole decode step: scores -> select -> rebuild -> attend.
 * out[H_q][d_h], idx[top_k], scores[L_c] (scores may be NULL). */
int s4r_oracle_decode_step(const s4r_oracle_problem *p, double *out,
                           int32_t *idx, double *scores);

/* Number of OpenMP threads the oracle runs on (1 when built without OpenMP). */
int s4r_oracle_threads(void);

/* Set the number of OpenMP threads for later calls (n >= 1); returns the
 * number now in effect.  Results do not depend on it: every output is a
 * sequential sum computed by one thread. */
int s4r_oracle_set_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
