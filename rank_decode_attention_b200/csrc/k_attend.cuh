// k_attend.cuh -- sparse reconstruction + exact attention.
//
// Eqs. 16-18 of S4R (review page, "Core claim"; "assumptions": sinks stay in
// full precision): the current query of head h (kv group g) attends over the
// n_sink sink tokens and the selected rows (top-k list + local window), whose
// keys and values are rebuilt from coefficients, k_hat = c_K B^K^T and
// v_hat = c_V B^V^T, restricted to the head's d_h columns of D'.
//
// The rebuild is evaluated in absorbed form, which is the same sum
// re-associated:  q . k_hat[g] = (q B^K[g]) . c_K   and
// sum_i p_i v_hat_i[g] = (sum_i p_i c_V,i) B^V[g]^T,  where B[g] are the d_h
// rows of the basis that belong to group g.  Nothing is rounded to the
// storage type; all arithmetic is fp32.
//
// attend_partial: CTA (split, g, b) runs an online softmax over a slice of
//   the selected rows for the G heads of group g and writes (m, l, acc[r_v]).
// attend_combine: CTA (h, b) merges the slices with the sink logits and maps
//   the latent accumulator back through B^V[g].
#pragma once
#include "common.cuh"
#include "k_topk.cuh"

namespace s4r {

constexpr int kAttThreads = 128;      // 4 warps
constexpr int kAttEntries = 64;       // selected rows per split
constexpr int kAttMaxGroup = 8;       // G <= 8
constexpr int kAttMaxRankLane = 8;    // rank / 32 <= 8

__host__ __device__ inline int64_t att_max_selected(const Shape &s) {
  return (int64_t)s.top_k + s.local_window;
}
__host__ __device__ inline int att_splits(const Shape &s) {
  return (int)ceil_div(att_max_selected(s) > 0 ? att_max_selected(s) : 1, kAttEntries);
}

// Row number of selected entry e (top-k list first, then the window).
__device__ __forceinline__ int64_t att_entry_row(const int32_t *idx_b, int64_t n_top, int64_t L,
                                                 int64_t n_win, int64_t e, int32_t n_sink) {
  if (e < n_top) return (int64_t)idx_b[e] - n_sink;
  return L - n_win + (e - n_top);
}

template <typename T>
__global__ void __launch_bounds__(kAttThreads)
attend_partial(Shape s, const int32_t *__restrict__ lengths, const int32_t *__restrict__ idx,
               const T *__restrict__ coeff_k, const T *__restrict__ coeff_v,
               const float *__restrict__ qt_all, float *__restrict__ part) {
  __shared__ float q_s[kAttMaxGroup][S4R_MAX_RANK];
  __shared__ float m_s[4][kAttMaxGroup], l_s[4][kAttMaxGroup];
  __shared__ float acc_s[4][kAttMaxGroup][S4R_MAX_RANK];
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = s.group, rk = s.rank_k, rv = s.rank_v;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t L = valid_length(lengths[b], s.cache_rows);
  const int64_t n_top = smin<int64_t>(s.top_k, n_candidates(L, s.local_window));
  const int64_t n_win = smin<int64_t>(s.local_window, L);
  const int64_t n_sel = n_top + n_win;
  const int64_t e0 = (int64_t)split * kAttEntries;
  const int64_t e1 = smin<int64_t>(n_sel, e0 + kAttEntries);
  for (int e = threadIdx.x; e < G * rk; e += blockDim.x) {
    const int j = e / rk, k = e - j * rk;
    q_s[j][k] = qt_all[((int64_t)b * s.n_heads_q + g * G + j) * rk + k];
  }
  __syncthreads();
  float m[kAttMaxGroup], l[kAttMaxGroup], acc[kAttMaxGroup][kAttMaxRankLane];
#pragma unroll
  for (int j = 0; j < kAttMaxGroup; ++j) {
    m[j] = -INFINITY; l[j] = 0.f;
#pragma unroll
    for (int u = 0; u < kAttMaxRankLane; ++u) acc[j][u] = 0.f;
  }
  const int32_t *idx_b = idx + (int64_t)b * s.top_k;
  const T *ckb = coeff_k + (int64_t)b * s.cache_rows * rk;
  const T *cvb = coeff_v + (int64_t)b * s.cache_rows * rv;
  for (int64_t e = e0 + wid; e < e1; e += 4) {
    const int64_t row = att_entry_row(idx_b, n_top, L, n_win, e, s.n_sink);
    if (row < 0 || row >= L) continue;  // idx entries come from the top-k kernel
    float ck[kAttMaxRankLane];
#pragma unroll
    for (int u = 0; u < kAttMaxRankLane; ++u) {
      const int k = lane + 32 * u;
      ck[u] = (k < rk) ? to_f(ckb[row * rk + k]) : 0.f;
    }
    float cv[kAttMaxRankLane];
#pragma unroll
    for (int u = 0; u < kAttMaxRankLane; ++u) {
      const int k = lane + 32 * u;
      cv[u] = (k < rv) ? to_f(cvb[row * rv + k]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kAttMaxGroup; ++j) {
      if (j >= G) break;
      float d = 0.f;
#pragma unroll
      for (int u = 0; u < kAttMaxRankLane; ++u) {
        const int k = lane + 32 * u;
        if (k < rk) d = fmaf(q_s[j][k], ck[u], d);
      }
      const float logit = warp_sum(d);
      const float nm = fmaxf(m[j], logit);
      const float scale = __expf(m[j] - nm);
      const float p = __expf(logit - nm);
      l[j] = l[j] * scale + p;
#pragma unroll
      for (int u = 0; u < kAttMaxRankLane; ++u) acc[j][u] = acc[j][u] * scale + p * cv[u];
      m[j] = nm;
    }
  }
  // Combine the 4 warps.
#pragma unroll
  for (int j = 0; j < kAttMaxGroup; ++j) {
    if (j >= G) break;
    if (lane == 0) { m_s[wid][j] = m[j]; l_s[wid][j] = l[j]; }
#pragma unroll
    for (int u = 0; u < kAttMaxRankLane; ++u) {
      const int k = lane + 32 * u;
      if (k < rv) acc_s[wid][j][k] = acc[j][u];
    }
  }
  __syncthreads();
  const int n_split = gridDim.x;
  for (int e = threadIdx.x; e < G * (rv + 2); e += blockDim.x) {
    const int j = e / (rv + 2), k = e - j * (rv + 2);
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, m_s[w][j]);
    float v = 0.f;
    if (k == 0) {
      v = M;
    } else {
      for (int w = 0; w < 4; ++w) {
        const float f = (m_s[w][j] == -INFINITY) ? 0.f : __expf(m_s[w][j] - M);
        v += f * ((k == 1) ? l_s[w][j] : acc_s[w][j][k - 2]);
      }
    }
    const int h = g * G + j;
    part[(((int64_t)b * s.n_heads_q + h) * n_split + split) * (rv + 2) + k] = v;
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
attend_combine(Shape s, const T *__restrict__ q, const T *__restrict__ basis_v,
               const T *__restrict__ sink_k, const T *__restrict__ sink_v,
               const float *__restrict__ part, float *__restrict__ out) {
  extern __shared__ float cs[];  // [rv] latent accumulator, then [n_sink] sink weights
  __shared__ float red[8];
  __shared__ float sh_M, sh_den;
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = s.group, g = h / G, dh = s.head_dim, rv = s.rank_v, Dp = s.d_model;
  const int ns = s.n_sink, n_split = att_splits(s);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  float *acc_s = cs;
  float *sw = cs + rv;
  const T *qh = q + (((int64_t)b * s.query_window + s.query_window - 1) * s.n_heads_q + h) * dh;
  const float *pb = part + ((int64_t)b * s.n_heads_q + h) * n_split * (rv + 2);
  // Sink logits, one warp per sink.
  const float qscale = rsqrtf((float)dh);
  for (int t = wid; t < ns; t += nw) {
    const T *kr = sink_k + ((int64_t)b * ns + t) * Dp + (int64_t)g * dh;
    float d = 0.f;
    for (int e = lane; e < dh; e += 32) d = fmaf(to_f(qh[e]), to_f(kr[e]), d);
    d = warp_sum(d);
    if (lane == 0) sw[t] = d * qscale;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    for (int t = 0; t < ns; ++t) M = fmaxf(M, sw[t]);
    for (int sp = 0; sp < n_split; ++sp) M = fmaxf(M, pb[sp * (rv + 2)]);
    float den = 0.f;
    for (int t = 0; t < ns; ++t) den += __expf(sw[t] - M);
    for (int sp = 0; sp < n_split; ++sp) {
      const float ms = pb[sp * (rv + 2)];
      if (ms != -INFINITY) den += pb[sp * (rv + 2) + 1] * __expf(ms - M);
    }
    sh_M = M;
    sh_den = den;
  }
  __syncthreads();
  const float M = sh_M;
  const float inv = (sh_den > 0.f) ? 1.f / sh_den : 0.f;
  for (int k = threadIdx.x; k < rv; k += blockDim.x) {
    float a = 0.f;
    for (int sp = 0; sp < n_split; ++sp) {
      const float ms = pb[sp * (rv + 2)];
      if (ms != -INFINITY) a += pb[sp * (rv + 2) + 2 + k] * __expf(ms - M);
    }
    acc_s[k] = a * inv;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < ns; t += blockDim.x) sw[t] = __expf(sw[t] - M) * inv;
  __syncthreads();
  (void)red;
  // out[h][e] = sum_k acc[k] B^V[g*dh + e][k] + sum_t w_t sink_v[t][g*dh + e]; one warp per e.
  const T *Bv = basis_v + (int64_t)b * Dp * rv;
  for (int e = wid; e < dh; e += nw) {
    const T *brow = Bv + (int64_t)(g * dh + e) * rv;
    float d = 0.f;
    for (int k = lane; k < rv; k += 32) d = fmaf(acc_s[k], to_f(brow[k]), d);
    d = warp_sum(d);
    if (lane == 0) {
      float sv = 0.f;
      for (int t = 0; t < ns; ++t)
        sv = fmaf(sw[t], to_f(sink_v[((int64_t)b * ns + t) * Dp + (int64_t)g * dh + e]), sv);
      out[((int64_t)b * s.n_heads_q + h) * dh + e] = d + sv;
    }
  }
}

// Rebuild rows explicitly: out[e][d] = sum_j C[rows[e]][j] B[d][j] (fp32).
template <typename T>
__global__ void __launch_bounds__(256)
reconstruct_kernel(const T *__restrict__ coeffs, int64_t n_rows_total, const T *__restrict__ basis,
                   int d_model, int rank, const int32_t *__restrict__ rows, int64_t n,
                   float *__restrict__ out) {
  __shared__ float c_s[S4R_MAX_RANK];
  const int64_t e = blockIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t row = rows[e];
  const bool ok = row >= 0 && row < n_rows_total;
  for (int j = threadIdx.x; j < rank; j += blockDim.x) c_s[j] = ok ? to_f(coeffs[row * rank + j]) : 0.f;
  __syncthreads();
  const int d0 = blockIdx.y * 64;
  for (int d = d0 + wid; d < min(d_model, d0 + 64); d += 8) {
    float acc = 0.f;
    for (int j = lane; j < rank; j += 32) acc = fmaf(c_s[j], to_f(basis[(int64_t)d * rank + j]), acc);
    acc = warp_sum(acc);
    if (lane == 0) out[e * d_model + d] = acc;
  }
}

}  // namespace s4r
