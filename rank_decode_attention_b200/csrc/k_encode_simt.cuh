// k_encode_simt.cuh -- encode C = S . B on CUDA cores (Eq. 3 of S4R, review
// page "What carries the argument": every non-sink token is stored as its
// coefficients in the rank-r basis).  fp32 accumulation, result rounded to the
// storage type with round-to-nearest-even.  Used for fp32 storage, for token
// counts too small for the tensor-core kernel, and for the per-problem append.
#pragma once
#include "common.cuh"
#include "k_topk.cuh"

namespace s4r {

constexpr int kEncTileM = 64, kEncTileN = 64, kEncTileK = 32;

template <typename T>
__global__ void __launch_bounds__(256)
encode_simt(const T *__restrict__ S, int64_t n, int64_t lds, const T *__restrict__ B, int d,
            int r, T *__restrict__ C, int64_t ldc) {
  __shared__ float s_s[kEncTileK][kEncTileM + 1];
  __shared__ float b_s[kEncTileK][kEncTileN + 1];
  const int64_t m0 = (int64_t)blockIdx.x * kEncTileM;
  const int n0 = blockIdx.y * kEncTileN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += kEncTileK) {
    for (int e = threadIdx.x; e < kEncTileM * kEncTileK; e += blockDim.x) {
      const int mm = e / kEncTileK, kk = e - mm * kEncTileK;
      const int64_t m = m0 + mm;
      const int k = k0 + kk;
      s_s[kk][mm] = (m < n && k < d) ? to_f(S[m * lds + k]) : 0.f;
    }
    for (int e = threadIdx.x; e < kEncTileK * kEncTileN; e += blockDim.x) {
      const int kk = e / kEncTileN, nn = e - kk * kEncTileN;
      const int k = k0 + kk, c = n0 + nn;
      b_s[kk][nn] = (k < d && c < r) ? to_f(B[(int64_t)k * r + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kEncTileK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = s_s[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = b_s[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 16 * i;
    if (m >= n) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx + 16 * j;
      if (c < r) C[m * ldc + c] = from_f<T>(acc[i][j]);
    }
  }
}

// Append: one token per problem, separate bases per problem, K and V.
// grid (batch, 2): block (b, 0) writes the key row, block (b, 1) the value
// row, both at row lengths[b].  The lengths are only read here; the next
// launch on the same stream (append_bump_lengths) increments them.
template <typename T>
__global__ void __launch_bounds__(256)
append_kernel(int d, int rk, int rv, int64_t cache_rows, const T *__restrict__ state_k,
              const T *__restrict__ state_v, const T *__restrict__ basis_k,
              const T *__restrict__ basis_v, T *__restrict__ coeff_k, T *__restrict__ coeff_v,
              const int32_t *__restrict__ len_in, uint32_t *__restrict__ status) {
  __shared__ float s_s[S4R_MAX_D_MODEL];
  const int b = blockIdx.x, which = blockIdx.y;
  const int r = which ? rv : rk;
  const T *st = (which ? state_v : state_k) + (int64_t)b * d;
  const T *B = (which ? basis_v : basis_k) + (int64_t)b * d * r;
  T *C = (which ? coeff_v : coeff_k) + (int64_t)b * cache_rows * r;
  const int64_t n = len_in[b];
  if (n < 0 || n >= cache_rows) {
    if (threadIdx.x == 0) set_status(status, kDevStatusCheck);
    return;
  }
  for (int e = threadIdx.x; e < d; e += blockDim.x) s_s[e] = to_f(st[e]);
  __syncthreads();
  for (int j = threadIdx.x; j < r; j += blockDim.x) {
    float acc = 0.f;
    for (int e = 0; e < d; ++e) acc = fmaf(s_s[e], to_f(B[(int64_t)e * r + j]), acc);
    C[n * r + j] = from_f<T>(acc);
  }
}

__global__ void append_bump_lengths(int batch, int64_t cache_rows, int32_t *__restrict__ lengths) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch && lengths[b] >= 0 && lengths[b] < cache_rows) lengths[b] += 1;
}

}  // namespace s4r
