// k_project.cuh -- query projection into the key basis.
//
// "Core claim" of the S4R review page: at decoding, queries are projected into
// the key subspace; the sliding query window is then scored in latent space
// (Eqs. 8-10).  One launch produces, per problem,
//   cq[R][r_k]   scoring rows C_Q, already multiplied by 1/sqrt(r_k), and
//   qt[H_q][r_k] the current query (window slot W-1) of every head projected
//                with the head_dim rows of its kv group's key-basis slice,
//                multiplied by 1/sqrt(head_dim) -- the absorbed form of the
//                exact-attention logits q . (c B^T) = (q B) . c.
// Output rows rho < R are scoring rows, rows R .. R+H_q-1 are the qt rows.
// Products of two storage values are exact in fp32; each 64-term chunk is
// summed in fp32 and the chunks in fp64, so the result is the fp64 dot
// product rounded once to fp32 (up to the chunk rounding).
#pragma once
#include "common.cuh"

namespace s4r {

constexpr int kProjRows = 8;    // output rows per CTA
constexpr int kProjCols = 32;   // rank columns per CTA
constexpr int kProjChunk = 64;  // D' rows staged per iteration

// Value of input row `rho` at model column d (0 outside the row's support).
template <typename T>
__device__ __forceinline__ float proj_input(const T *q, const Shape &s, int rho, int d) {
  const int dh = s.head_dim, G = s.group, Hq = s.n_heads_q;
  const int g = d / dh, t = d - g * dh;
  int w, h;
  if (rho < s.n_rows) {
    if (s.row_mode == S4R_ROWS_CONCAT) {
      w = rho / G;
      h = g * G + (rho - w * G);
    } else {
      w = rho / Hq;
      h = rho - w * Hq;
      if (h / G != g) return 0.f;
    }
  } else {
    w = s.query_window - 1;
    h = rho - s.n_rows;
    if (h / G != g) return 0.f;
  }
  return to_f(q[((int64_t)w * Hq + h) * dh + t]);
}

template <typename T>
__global__ void __launch_bounds__(kProjRows * kProjCols)
project_kernel(Shape s, const T *__restrict__ q, const T *__restrict__ basis_k,
               float *__restrict__ cq, float *__restrict__ qt, double *__restrict__ row_sum,
               unsigned long long *__restrict__ barrier) {
  __shared__ float qs[kProjRows][kProjChunk + 1];
  __shared__ float bs[kProjChunk][kProjCols + 1];
  const int b = blockIdx.z;
  const int row0 = blockIdx.x * kProjRows, col0 = blockIdx.y * kProjCols;
  const int tx = threadIdx.x % kProjCols, ty = threadIdx.x / kProjCols;
  const int n_out = s.n_rows + s.n_heads_q;
  const int r = s.rank_k, Dp = s.d_model;
  const T *qb = q + (int64_t)b * s.query_window * s.n_heads_q * s.head_dim;
  const T *Bb = basis_k + (int64_t)b * Dp * r;
  // Reset the per-call accumulators of the tensor-core scoring kernel.
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    for (int e = threadIdx.x; e < s.n_rows; e += blockDim.x) row_sum[(int64_t)b * s.n_rows + e] = 0.0;
    if (b == 0 && threadIdx.x == 0) *barrier = 0ull;
  }
  double acc = 0.0;
  for (int d0 = 0; d0 < Dp; d0 += kProjChunk) {
    for (int e = threadIdx.x; e < kProjRows * kProjChunk; e += blockDim.x) {
      const int rr = e / kProjChunk, dd = e % kProjChunk;
      const int rho = row0 + rr, d = d0 + dd;
      qs[rr][dd] = (rho < n_out && d < Dp) ? proj_input(qb, s, rho, d) : 0.f;
    }
    for (int e = threadIdx.x; e < kProjChunk * kProjCols; e += blockDim.x) {
      const int dd = e / kProjCols, cc = e % kProjCols;
      const int d = d0 + dd, c = col0 + cc;
      bs[dd][cc] = (d < Dp && c < r) ? to_f(Bb[(int64_t)d * r + c]) : 0.f;
    }
    __syncthreads();
    float part = 0.f;
#pragma unroll 8
    for (int dd = 0; dd < kProjChunk; ++dd) part = fmaf(qs[ty][dd], bs[dd][tx], part);
    acc += (double)part;
    __syncthreads();
  }
  const int rho = row0 + ty, c = col0 + tx;
  if (rho >= n_out || c >= r) return;
  if (rho < s.n_rows) {
    cq[((int64_t)b * s.n_rows + rho) * r + c] = (float)(acc / sqrt((double)r));
  } else {
    const int h = rho - s.n_rows;
    qt[((int64_t)b * s.n_heads_q + h) * r + c] = (float)(acc / sqrt((double)s.head_dim));
  }
}

}  // namespace s4r
