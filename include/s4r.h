/*
 * s4r.h -- C ABI of libs4r: S4R compressed-KV decode on NVIDIA B200 (sm_100a).
 *
 * The operations are those of "S^4R: Selective Sampling, Subspaces, and
 * Sparse Reconstruction for Compressed Long-Context KV Caching"
 * (arXiv 2608.00528), as its review page on pith.science states them:
 *   - every non-sink token is stored as rank-r coefficients c = s . B
 *     ("What carries the argument", Eq. 3);
 *   - a decode step projects a sliding window of queries into the key basis,
 *     scores every cached key coefficient in latent space with a softmax
 *     (major comment 2, §3.2.2, Eqs. 8-10), keeps the local window plus the
 *     top-k earlier positions (Eqs. 13-15), rebuilds only those rows from
 *     their coefficients and runs exact attention together with the
 *     uncompressed sink tokens (Eqs. 16-18).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers unless a comment says "host".
 *     Every device pointer must be 16-byte aligned.
 *   - The caller owns every buffer.  The library allocates no device memory,
 *     keeps no per-call state between calls and may be called from several
 *     host threads on different streams (each call with its own workspace).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work; none synchronises, except
 *     s4r_read_device_status.
 *   - The kernels of consecutive decode calls on one stream overlap their
 *     start-up (programmatic dependent launch): a call's first kernel may
 *     begin, and read the call's inputs (queries, coefficient caches, bases,
 *     sinks, lengths), while the previous decode call's last kernel is still
 *     running; it touches the workspace and the outputs only after that
 *     kernel has completed.  So the inputs of a call must be complete when
 *     it is enqueued: written by earlier calls or copies, or by kernels that
 *     do not release their dependents early.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and returned as S4R_ERR_INVALID_ARG / S4R_ERR_UNSUPPORTED /
 *     S4R_ERR_WORKSPACE.  A failed launch returns S4R_ERR_CUDA.  Conditions
 *     only the device can see (a full cache on append, a length beyond the
 *     cache capacity, a bounded wait that gave up) set a sticky status word
 *     in the workspace, which s4r_read_device_status returns; the kernels
 *     then skip the offending work instead of touching memory out of bounds.
 *
 * Layouts (row-major, innermost index last).  D' = n_heads_kv * head_dim,
 * G = n_heads_q / n_heads_kv; query head h belongs to kv group g = h / G and
 * uses columns g*head_dim .. (g+1)*head_dim-1 of D'.  Coefficient row i of a
 * problem stores absolute token position n_sink + i; the first n_sink tokens
 * are the uncompressed sinks.
 */
#ifndef S4R_H
#define S4R_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  S4R_OK = 0,
  S4R_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, inconsistent shape */
  S4R_ERR_UNSUPPORTED = 2,  /* valid request outside the supported range */
  S4R_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  S4R_ERR_TIMEOUT = 4,      /* device status: a bounded device-side wait gave up */
  S4R_ERR_DEVICE = 5,       /* device status: a device-side check failed */
  S4R_ERR_WORKSPACE = 6     /* workspace pointer null or smaller than required */
} s4r_status;

typedef enum { S4R_F32 = 0, S4R_BF16 = 1 } s4r_dtype;

/* How the query window forms scoring rows (Eqs. 8-10).
 * CONCAT (default): W*G rows; row (w, j) concatenates query head g*G + j of
 *   every kv group g into one D'-vector, projected with the whole key basis.
 * PER_HEAD: W*H_q rows; row (w, h) projects query head h with the head_dim
 *   rows of the key basis that belong to its kv group. */
typedef enum { S4R_ROWS_CONCAT = 0, S4R_ROWS_PER_HEAD = 1 } s4r_row_mode;

/* Pooling of the candidate scores before selection (pool_kernel = odd kappa
 * > 1; "free parameters": kernel 7, from SnapKV).  Stride 1, same padding,
 * over the candidates only; neighbours outside the candidates are left out.
 * MAX: the largest neighbour score.  AVG: the mean of the in-range
 * neighbour scores (their sum in fp32, in position order, divided by their
 * count). */
typedef enum { S4R_POOL_MAX = 0, S4R_POOL_AVG = 1 } s4r_pool_mode;

/* Supported range (S4R_ERR_UNSUPPORTED outside it). */
#define S4R_MAX_D_MODEL 1024    /* D' */
#define S4R_MAX_RANK 256        /* rank_k, rank_v; multiples of 8 */
#define S4R_MAX_HEAD_DIM 256    /* multiple of 8 */
#define S4R_MAX_SCORE_ROWS 512  /* W*G (CONCAT) or W*H_q (PER_HEAD) */
#define S4R_MAX_POOL_KERNEL 63  /* odd */
#define S4R_MAX_GROUP 8         /* G = n_heads_q / n_heads_kv */
#define S4R_MAX_SINKS 16        /* n_sink */
#define S4R_MAX_SELECTED 8192   /* top_k + local_window */
#define S4R_MAX_BASIS_SAMPLE 1048576  /* n_sample T' of s4r_build_basis */

/* ------------------------------------------------------------------ encode */

/* Encode token states into coefficients, C = S . B ("What carries the
 * argument", Eq. 3): coeffs[t][j] = sum_d states[t][d] * basis[d][j].
 *   states  [n_tokens][d_model], row stride states_ld elements (>= d_model)
 *   basis   [d_model][rank], contiguous
 *   coeffs  [n_tokens][rank], row stride coeffs_ld elements (>= rank)
 * All three have type `dtype`; accumulation is fp32 and the result is
 * rounded to `dtype` (round to nearest even).  n_tokens == 0 is a no-op.
 * Strides must keep every row 16-byte aligned. */
s4r_status s4r_encode(const void *states, int64_t n_tokens, int64_t states_ld,
                      const void *basis, int32_t d_model, int32_t rank,
                      void *coeffs, int64_t coeffs_ld, s4r_dtype dtype, void *stream);

/* Encode two token sets against their own bases in one launch: the K and V
 * halves of a prompt (Eq. 3, "What carries the argument"), for p = 0, 1:
 *   coeffs_p[t][j] = sum_d states_p[t][d] * basis_p[d][j],  t < n_tokens.
 * Each (states_p, basis_p, coeffs_p) follows the layout, type, rounding and
 * alignment rules of s4r_encode; both share n_tokens, the strides, d_model
 * and rank.  The result equals two s4r_encode calls (the tensor-core path
 * runs both in one persistent grid, so the second problem's tiles fill the
 * SMs the first leaves idle).  Inputs and outputs stay owned by the caller. */
s4r_status s4r_encode2(const void *states0, const void *states1, int64_t n_tokens, int64_t states_ld,
                       const void *basis0, const void *basis1, int32_t d_model, int32_t rank,
                       void *coeffs0, void *coeffs1, int64_t coeffs_ld, s4r_dtype dtype, void *stream);

/* Append one new token per problem to the coefficient caches (Eq. 3 applied
 * to the token a decode step adds).  For each problem b, with n = lengths[b]
 * read on the device:
 *   coeff_k[b][n] = state_k[b] . basis_k[b],  coeff_v[b][n] = state_v[b] . basis_v[b],
 *   then lengths[b] = n + 1.
 * If n >= cache_rows the problem is skipped and the device status
 * (S4R_ERR_DEVICE) is set in `status_workspace` (may be NULL: skip only). */
typedef struct {
  int32_t batch, d_model, rank_k, rank_v;
  s4r_dtype dtype;
  int64_t cache_rows;                 /* row capacity of each problem's caches */
  const void *state_k, *state_v;      /* [batch][d_model] */
  const void *basis_k, *basis_v;      /* [batch][d_model][rank] */
  void *coeff_k, *coeff_v;            /* [batch][cache_rows][rank] */
  int32_t *lengths;                   /* [batch] device, read and incremented */
  void *status_workspace;             /* a decode workspace (its status word), or NULL */
} s4r_append_args;

s4r_status s4r_append(const s4r_append_args *args, void *stream);

/* ------------------------------------------------------------------ bases */

/* Build the low-rank bases at prefill ("What carries the argument" and the
 * Referee Report's summary, Eqs. 1-2; "Core claim" for the sample): for each
 * problem, the top-r right singular vectors of a sampled, token-wise
 * normalised set of its non-sink states.  With L = lengths[p] (read on the
 * device) and n = min(n_sample, L - n_sink) sample rows:
 *   - the last (7n + 5) div 10 rows L-1, L-2, ... (0.7 n rounded half up)
 *     and n_u = n - that many rows s + floor(j * span / n_u), j < n_u,
 *     spread over the older non-sink rows (span = L - s - recent rows);
 *   - every sampled row scaled to unit Euclidean norm (zero rows stay zero);
 *   - basis column k = right singular vector of the k-th largest singular
 *     value sigma[k], signed so that its largest-magnitude entry (lowest
 *     index on ties) is positive.
 * Arithmetic is fp64 throughout (the Gram matrix of the smaller side of the
 * sample and its eigenvectors by parallel cyclic Jacobi rotations); the
 * library owns no memory, so the caller passes a workspace of
 * s4r_basis_workspace_bytes() bytes whose first word is the sticky device
 * status (zero it once with s4r_workspace_init; read it with
 * s4r_read_device_status).  The status is set (S4R_ERR_DEVICE) when a
 * length lies outside [0, state_rows], when a sample has fewer than r rows
 * or rank below r (a kept sigma^2 at or below 1e-13 of the largest), or when
 * the rotations do not settle within 30 sweeps; S4R_ERR_TIMEOUT when a
 * grid-wide wait gave up.  The outputs of such a problem are then not a
 * basis. */
typedef struct {
  int32_t n_problems;     /* independent (sequence, layer, K or V) problems */
  int32_t d_model;        /* D' (<= S4R_MAX_D_MODEL) */
  int32_t rank;           /* r (<= min(n_sample, D', S4R_MAX_RANK)) */
  int32_t n_sink;         /* s: leading rows never sampled */
  int32_t n_sample;       /* T' (<= S4R_MAX_BASIS_SAMPLE) */
  s4r_dtype dtype;        /* type of states and basis_out */
  int64_t state_rows;     /* rows per problem in states (>= every length) */
  const int32_t *lengths; /* [n_problems] prompt length L of each problem */
  const void *states;     /* [n_problems][state_rows][D'] token states */
  void *basis_out;        /* [n_problems][D'][r] in dtype (fp64 -> fp32 -> dtype,
                             nearest even), or NULL */
  double *basis_f64;      /* [n_problems][D'][r] fp64, or NULL (not both NULL) */
  double *sigma;          /* [n_problems][r] singular values, or NULL */
  void *workspace;        /* s4r_basis_workspace_bytes(args) bytes */
  size_t workspace_bytes;
} s4r_basis_args;

/* Workspace bytes for these arguments (0 if they are invalid). */
size_t s4r_basis_workspace_bytes(const s4r_basis_args *args);

/* Enqueue the basis build (six kernels, one of them a cooperative launch).
 * Host-side argument errors: S4R_ERR_INVALID_ARG (null or misaligned
 * pointers, rank above n_sample or D'), S4R_ERR_UNSUPPORTED (sizes above the
 * limits), S4R_ERR_WORKSPACE. */
s4r_status s4r_build_basis(const s4r_basis_args *args, void *stream);

/* ------------------------------------------------------------------ decode */

typedef struct {
  int32_t batch;                      /* independent (sequence, layer) problems */
  int32_t n_heads_q, n_heads_kv, head_dim;
  int32_t rank_k, rank_v;
  int32_t n_sink;                     /* s: uncompressed sink tokens per problem */
  int32_t local_window;               /* w: newest coefficient rows always kept */
  int32_t top_k;                      /* k: global positions chosen before the window */
  int32_t query_window;               /* W: query rows scored per step */
  int32_t pool_kernel;                /* 1 = off; odd kappa = pool candidate scores */
  int32_t pool_mode;                  /* s4r_pool_mode (read when pool_kernel > 1) */
  int32_t row_mode;                   /* s4r_row_mode */
  s4r_dtype dtype;                    /* storage type of q, coefficients, bases, sinks */
  int64_t cache_rows;                 /* row capacity (stride) of the coefficient caches */
  const int32_t *lengths;             /* [batch] device: L_c, coefficient rows in use */
  const void *q;                      /* [batch][W][H_q][head_dim]; slot W-1 = current query */
  const void *coeff_k, *coeff_v;      /* [batch][cache_rows][rank_k | rank_v] */
  const void *basis_k, *basis_v;      /* [batch][D'][rank_k | rank_v] */
  const void *sink_k, *sink_v;        /* [batch][n_sink][D'] */
  float *out;                         /* [batch][H_q][head_dim] attention output */
  int32_t *idx;                       /* [batch][top_k] chosen absolute positions,
                                         ascending, -1 padded (window not listed) */
  float *scores;                      /* optional [batch][cache_rows] latent scores, or NULL */
  void *workspace;                    /* device scratch, see s4r_decode_workspace_bytes */
  size_t workspace_bytes;
  void *profile_events[2];            /* optional cudaEvent_t pair (or NULL): recorded on
                                         `stream` right before and right after the
                                         latent-scoring kernels, for timing them; under
                                         stream capture they become external event
                                         record nodes of the graph */
} s4r_decode_args;

/* Bytes of device workspace s4r_decode_step needs for these arguments (only
 * the shape fields are read).  Returns 0 if the shape is invalid. */
size_t s4r_decode_workspace_bytes(const s4r_decode_args *args);

/* Number of kernel launches one s4r_decode_step with these arguments
 * enqueues (0 if the shape is invalid). */
int32_t s4r_decode_kernel_launches(const s4r_decode_args *args);

/* Prepare a freshly allocated workspace: zeroes all of it (status word,
 * counters and accumulators that the kernels reuse and leave zeroed after
 * each call).  Call once per workspace allocation, before its first use. */
s4r_status s4r_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* One decode step for every problem of the batch:
 *   1. C_Q = Q' . B^K for the query window (rows per row_mode);
 *   2. Z = C_Q . C_K^T / sqrt(rank_k), softmax of every row over the L_c
 *      coefficient rows, score[i] = sum of the rows' probabilities (Eqs. 8-10);
 *   3. idx = the top_k rows among 0 .. L_c-w-1 by score (pooled by
 *      pool_mode when pool_kernel > 1), equal scores -> lower position
 *      (Eqs. 13-15);
 *   4. for every query head h, exact attention of q[W-1][h] over the sinks,
 *      the chosen rows and the last w rows, with keys c_K . B^K^T and values
 *      c_V . B^V^T restricted to the head's kv group, logits scaled by
 *      1/sqrt(head_dim) (Eqs. 16-18).  Rebuilt rows are kept in fp32.
 * Arithmetic is fp32 whatever the storage type. */
s4r_status s4r_decode_step(const s4r_decode_args *args, void *stream);

/* ------------------------------------------------- decode without alloc */

/* Library extension: the S4R paper has no counterpart to this entry point.
 *
 * The same decode step as s4r_decode_step, for callers that cannot allocate
 * or own device memory for a workspace (a host program that manages no
 * device memory, or an engine that has handed all free HBM to its cache pool
 * and may not allocate while serving).  Instead of args->workspace (ignored,
 * may be NULL) it uses a scratch array of S4R_NOALLOC_SCRATCH_BYTES compiled
 * into the library, one per device.  It allocates nothing.
 *   - Shapes whose s4r_decode_workspace_bytes exceeds
 *     S4R_NOALLOC_SCRATCH_BYTES are rejected with S4R_ERR_UNSUPPORTED before
 *     anything is enqueued; s4r_last_error names both sizes.
 *   - The first call on a device (current device at call time) looks up the
 *     array and zeroes it synchronously; make that first call before any
 *     stream capture or other work that must not be synchronised.
 *   - Every call on a device shares the one array.  Calls that may overlap
 *     in time (other streams or host threads) race on it and give wrong
 *     results; order them on one stream or synchronise between them.
 *   - Device-side conditions (a bounded wait that gave up, a bad length) go
 *     to the library-wide status of the device: read them with
 *     s4r_read_device_status(NULL, stream). */
#define S4R_NOALLOC_SCRATCH_BYTES (4u << 20)
s4r_status s4r_decode_step_noalloc(const s4r_decode_args *args, void *stream);

/* ----------------------------------------------------------- reconstruct */

/* Rebuild selected rows from coefficients, out[e][d] = sum_j coeffs[rows[e]][j]
 * * basis[d][j] (Eq. 16).  coeffs [n_rows_total][rank] and basis
 * [d_model][rank] have type `dtype`; rows [n] device int32 row numbers (a
 * row < 0 or >= n_rows_total yields a zero output row); out [n][d_model]
 * fp32. */
s4r_status s4r_reconstruct(const void *coeffs, int64_t n_rows_total, const void *basis,
                           int32_t d_model, int32_t rank, const int32_t *rows, int64_t n,
                           float *out, s4r_dtype dtype, void *stream);

/* ------------------------------------------------------------------ status */

/* Synchronise `stream`, then return the sticky device status of `workspace`
 * (S4R_OK, S4R_ERR_TIMEOUT or S4R_ERR_DEVICE); S4R_ERR_CUDA if the
 * synchronisation itself failed.  workspace == NULL reads the library-wide
 * status of the current device, which the kernels that take no workspace
 * (encode, reconstruct) report to. */
s4r_status s4r_read_device_status(const void *workspace, void *stream);

/* Reset the device status word of `workspace` (stream-ordered), or the
 * library-wide word of the current device when workspace == NULL (this
 * form synchronises `stream`). */
s4r_status s4r_clear_device_status(void *workspace, void *stream);

/* Testing hook for the device-side bounded waits; the S4R paper has no
 * counterpart.  Every spin-wait of the kernels (mbarrier waits, grid-wide
 * barriers) gives up after a limit, sets S4R_ERR_TIMEOUT in the device
 * status and lets the kernel finish without it (the call's results are then
 * not defined, but nothing hangs and the context stays usable).  This call
 * sets, for the current device:
 *   - limit_cycles: the limit in SM clock cycles (<= 0: the default, about
 *     2 s);
 *   - unreachable_barrier: when non-zero, the grid-wide barrier of the
 *     latent-scoring kernel waits for one arrival more than its grid has,
 *     so it always runs out after the limit.
 * It synchronises the device (cudaMemcpyToSymbol); do not call it while
 * other work of this library runs.  S4R_ERR_CUDA if the copy fails. */
s4r_status s4r_debug_waits(int64_t limit_cycles, int32_t unreachable_barrier);

/* Static description of a status code. */
const char *s4r_status_string(s4r_status status);

/* Human-readable description of the last S4R_ERR_CUDA returned on the
 * calling host thread (which step failed and the CUDA error name); "" if
 * none.  The string stays valid until the next failing call on the thread. */
const char *s4r_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t s4r_version(void);

#ifdef __cplusplus
}
#endif
#endif /* S4R_H */
