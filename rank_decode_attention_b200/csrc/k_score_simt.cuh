// k_score_simt.cuh -- latent relevance scoring on CUDA cores, fp64 accumulation.
//
// Eqs. 8-10 of S4R (review page, major comment 2, §3.2.2):
//   z[row][i]  = C_Q[row] . C_K[i] / sqrt(r)    (1/sqrt(r) is folded into cq)
//   P[row][i]  = exp(z - M_row) / l_row         (softmax over all L_c rows)
//   score[i]   = sum_row P[row][i]
// Three launches: per-tile row statistics, a merge of the tile statistics
// into (M_row, l_row), and a second pass that recomputes z and writes the
// scores.  Every logit, exponential and sum is float64; this is the precise
// CUDA-core path, used for fp32 storage and as the fallback of the tensor-core
// path.
#pragma once
#include "common.cuh"

namespace s4r {

constexpr int kScoreTile = 64;      // positions per CTA
constexpr int kScoreRowChunk = 64;  // scoring rows staged at once
constexpr int kScoreThreads = 256;  // 16 x 16, each thread 4 positions x 4 rows

struct ScoreSmem {
  // c tile [64][r+1] fp32, cq chunk [64][r+1] fp32, z staging [64][65] fp64
  static size_t bytes(int r) {
    return sizeof(float) * (size_t)kScoreTile * (r + 1) * 2 + sizeof(double) * kScoreRowChunk * 65;
  }
};

// Load the coefficient tile (zero past L) and compute z for one 64-row chunk.
// z_s[row][pos] receives float64 logits of the chunk.
template <typename T>
__device__ __forceinline__ void score_tile_logits(const float *c_s, float *cq_s, double *z_s,
                                                  const float *__restrict__ cq, int r,
                                                  int row0, int n_rows) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int ld = r + 1;
  for (int e = threadIdx.x; e < kScoreRowChunk * r; e += blockDim.x) {
    const int rr = e / r, k = e - rr * r;
    cq_s[rr * ld + k] = (row0 + rr < n_rows) ? cq[(int64_t)(row0 + rr) * r + k] : 0.f;
  }
  __syncthreads();
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  for (int k = 0; k < r; ++k) {
    double a[4], bq[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = (double)c_s[(ty + 16 * i) * ld + k];
#pragma unroll
    for (int j = 0; j < 4; ++j) bq[j] = (double)cq_s[(tx + 16 * j) * ld + k];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], bq[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) z_s[(tx + 16 * j) * 65 + (ty + 16 * i)] = acc[i][j];
  __syncthreads();
}

template <typename T>
__device__ __forceinline__ void load_coeff_tile(float *c_s, const T *__restrict__ ck, int r,
                                                int64_t pos0, int64_t L) {
  const int ld = r + 1;
  constexpr int V = Vec16<T>::n;
  const int vpr = r / V;  // 16-byte vectors per row (r % 8 == 0)
  for (int e = threadIdx.x; e < kScoreTile * vpr; e += blockDim.x) {
    const int p = e / vpr, v = e - p * vpr;
    float tmp[V];
    if (pos0 + p < L) {
      load16(ck + (pos0 + p) * r + v * V, tmp);
    } else {
#pragma unroll
      for (int u = 0; u < V; ++u) tmp[u] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < V; ++u) c_s[p * ld + v * V + u] = tmp[u];
  }
}

// Pass 1: per (tile, row) max and sum of exp(z - tile max), float64.
template <typename T>
__global__ void __launch_bounds__(kScoreThreads)
score_stats_simt(Shape s, const int32_t *__restrict__ lengths, const T *__restrict__ coeff_k,
                 const float *__restrict__ cq_all, double *__restrict__ tstat) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int b = blockIdx.y, r = s.rank_k;
  const int64_t L = lengths[b];
  const int64_t pos0 = (int64_t)blockIdx.x * kScoreTile;
  if (L <= 0 || L > s.cache_rows || pos0 >= L) return;
  float *c_s = reinterpret_cast<float *>(smem_raw);
  float *cq_s = c_s + kScoreTile * (r + 1);
  double *z_s = reinterpret_cast<double *>(cq_s + kScoreRowChunk * (r + 1));
  load_coeff_tile(c_s, coeff_k + (int64_t)b * s.cache_rows * r, r, pos0, L);
  const int n_valid = (int)smin<int64_t>(kScoreTile, L - pos0);
  const int64_t n_tiles = ceil_div(s.cache_rows, kScoreTile);
  for (int row0 = 0; row0 < s.n_rows; row0 += kScoreRowChunk) {
    __syncthreads();
    score_tile_logits<T>(c_s, cq_s, z_s, cq_all + (int64_t)b * s.n_rows * r, r, row0, s.n_rows);
    // 4 threads per row, 16 positions each.
    const int rr = threadIdx.x >> 2, part = threadIdx.x & 3;
    double m = -INFINITY;
    for (int p = part * 16; p < part * 16 + 16; ++p)
      if (p < n_valid) m = fmax(m, z_s[rr * 65 + p]);
    m = fmax(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmax(m, __shfl_xor_sync(0xffffffffu, m, 2));
    double l = 0.0;
    for (int p = part * 16; p < part * 16 + 16; ++p)
      if (p < n_valid) l += exp(z_s[rr * 65 + p] - m);
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (part == 0 && row0 + rr < s.n_rows) {
      double *t = tstat + (((int64_t)b * n_tiles + blockIdx.x) * s.n_rows + row0 + rr) * 2;
      t[0] = m;
      t[1] = l;
    }
  }
}

// Merge tile statistics into row statistics (M, l).  One warp per row, the
// lanes take tiles round-robin and the partial results are combined in a
// fixed shuffle order, so the result is deterministic.
__global__ void score_merge(Shape s, const int32_t *__restrict__ lengths,
                            const double *__restrict__ tstat, double *__restrict__ rstat) {
  const int b = blockIdx.y;
  const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= s.n_rows) return;
  const int64_t L = lengths[b];
  const int64_t n_tiles = ceil_div(s.cache_rows, kScoreTile);
  const int64_t used = (L > 0 && L <= s.cache_rows) ? ceil_div(L, kScoreTile) : 0;
  double m = -INFINITY, l = 0.0;
  for (int64_t t = lane; t < used; t += 32) {
    const double *st = tstat + (((int64_t)b * n_tiles + t) * s.n_rows + row) * 2;
    const double tm = st[0], tl = st[1];
    const double nm = fmax(m, tm);
    l = l * exp(m - nm) + tl * exp(tm - nm);
    m = nm;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double om = __shfl_xor_sync(0xffffffffu, m, o);
    const double ol = __shfl_xor_sync(0xffffffffu, l, o);
    const double nm = fmax(m, om);
    l = (nm == -INFINITY) ? 0.0 : l * exp(m - nm) + ol * exp(om - nm);
    m = nm;
  }
  if (lane == 0) {
    rstat[((int64_t)b * s.n_rows + row) * 2] = m;
    rstat[((int64_t)b * s.n_rows + row) * 2 + 1] = l;
  }
}

// Pass 2: recompute z and write score[i] = sum_row exp(z - M_row) / l_row.
template <typename T>
__global__ void __launch_bounds__(kScoreThreads)
score_final_simt(Shape s, const int32_t *__restrict__ lengths, const T *__restrict__ coeff_k,
                 const float *__restrict__ cq_all, const double *__restrict__ rstat,
                 float *__restrict__ scores) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int b = blockIdx.y, r = s.rank_k;
  const int64_t L = lengths[b];
  const int64_t pos0 = (int64_t)blockIdx.x * kScoreTile;
  if (L <= 0 || L > s.cache_rows || pos0 >= L) return;
  float *c_s = reinterpret_cast<float *>(smem_raw);
  float *cq_s = c_s + kScoreTile * (r + 1);
  double *z_s = reinterpret_cast<double *>(cq_s + kScoreRowChunk * (r + 1));
  __shared__ double sc_s[kScoreTile];
  load_coeff_tile(c_s, coeff_k + (int64_t)b * s.cache_rows * r, r, pos0, L);
  if (threadIdx.x < kScoreTile) sc_s[threadIdx.x] = 0.0;
  const int n_valid = (int)smin<int64_t>(kScoreTile, L - pos0);
  for (int row0 = 0; row0 < s.n_rows; row0 += kScoreRowChunk) {
    __syncthreads();
    score_tile_logits<T>(c_s, cq_s, z_s, cq_all + (int64_t)b * s.n_rows * r, r, row0, s.n_rows);
    // 4 threads per position, 16 rows each, in row order.
    const int p = threadIdx.x >> 2, part = threadIdx.x & 3;
    double acc = 0.0;
    for (int rr = part * 16; rr < part * 16 + 16; ++rr) {
      const int row = row0 + rr;
      if (row < s.n_rows) {
        const double M = rstat[((int64_t)b * s.n_rows + row) * 2];
        const double l = rstat[((int64_t)b * s.n_rows + row) * 2 + 1];
        acc += exp(z_s[rr * 65 + p] - M) / l;
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (part == 0) sc_s[p] += acc;
  }
  __syncthreads();
  if (threadIdx.x < n_valid)
    scores[(int64_t)b * s.cache_rows + pos0 + threadIdx.x] = (float)sc_s[threadIdx.x];
}

}  // namespace s4r
