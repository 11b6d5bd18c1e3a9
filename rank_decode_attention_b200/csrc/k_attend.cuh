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
// One launch, CTA (split, g, problem), 256 threads:
//   1. cp.async the split's selected C_K / C_V rows (<= 64) into shared memory;
//   2. logits of the G heads of group g, their softmax partials (max, sum) and
//      the latent value sums acc[j][:] = sum_e p[j][e] c_V[e];
//   3. write the partial; the last CTA of the group (atomic ticket) merges all
//      splits with the sink logits, maps acc through B^V[g] and writes out.
#pragma once
#include "common.cuh"
#include "k_topk.cuh"
#include "umma.cuh"

namespace s4r {

constexpr int kAttThreads = 256;      // 8 warps
constexpr int kAttMaxSplits = 128;    // (top_k + local_window) <= 128 * 64
constexpr int kAttEntries = 64;       // selected rows per split
constexpr int kAttMaxGroup = 8;       // G <= 8
constexpr int kAttMaxSinks = 16;      // sinks merged by the combining CTA

__host__ __device__ inline int64_t att_max_selected(const Shape &s) {
  return (int64_t)s.top_k + s.local_window;
}
__host__ __device__ inline int att_splits(const Shape &s) {
  return (int)ceil_div(att_max_selected(s) > 0 ? att_max_selected(s) : 1, kAttEntries);
}
// Row pitch (elements) of staged rows: 16-byte multiples whose 4-byte-word
// stride is 4 (mod 8), so the 16-byte reads of 8 consecutive rows fall in
// distinct bank quads.
__host__ __device__ inline int att_pitch(int n, int esize) {
  int words = (n * esize) / 4;
  while (words % 8 != 4) words += 4;
  return words * 4 / esize;
}
__host__ __device__ inline size_t att_stage_bytes(const Shape &s, int esize) {
  const size_t rows = (size_t)kAttEntries * (att_pitch(s.rank_k, esize) + att_pitch(s.rank_v, esize)) * esize;
  const size_t bv = (size_t)s.head_dim * att_pitch(s.rank_v, esize) * esize;
  return rows > bv ? rows : bv;
}
__host__ inline size_t att_smem_bytes(const Shape &s, int esize) {
  return att_stage_bytes(s, esize) +
         sizeof(float) * (size_t)(kAttMaxGroup * s.rank_k + kAttMaxGroup * kAttEntries + 4 * kAttMaxGroup +
                                  kAttMaxGroup * s.rank_v + kAttMaxGroup * kAttMaxSinks +
                                  kAttMaxGroup * kAttMaxSplits);
}

// Row number of selected entry e (top-k list first, then the window).
__device__ __forceinline__ int64_t att_entry_row(const int32_t *idx_b, int64_t n_top, int64_t L,
                                                 int64_t n_win, int64_t e, int32_t n_sink) {
  if (e < n_top) return (int64_t)idx_b[e] - n_sink;
  return L - n_win + (e - n_top);
}

// Dot product of n (a multiple of 8) fp32 values with n storage values, 16-byte reads.
template <typename T>
__device__ __forceinline__ float dot_f32_store(const float *a, const T *x, int n) {
  constexpr int V = Vec16<T>::n;
  float acc = 0.f;
  for (int k = 0; k < n; k += V) {
    float xv[V];
    load16(x + k, xv);
#pragma unroll
    for (int u = 0; u < V; ++u) acc = fmaf(a[k + u], xv[u], acc);
  }
  return acc;
}

template <typename T>
__global__ void __launch_bounds__(kAttThreads)
attend_kernel(Shape s, const int32_t *__restrict__ lengths, const int32_t *__restrict__ idx,
              const T *__restrict__ coeff_k, const T *__restrict__ coeff_v, const float *__restrict__ qt_all,
              const T *__restrict__ q, const T *__restrict__ basis_v, const T *__restrict__ sink_k,
              const T *__restrict__ sink_v, float *__restrict__ part, unsigned int *__restrict__ tickets,
              float *__restrict__ out) {
  extern __shared__ __align__(16) unsigned char att_smem[];
  constexpr int V = Vec16<T>::n;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int n_split = gridDim.x;
  const int G = s.group, rk = s.rank_k, rv = s.rank_v, dh = s.head_dim, Dp = s.d_model, ns = s.n_sink;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int pk = att_pitch(rk, sizeof(T)), pv = att_pitch(rv, sizeof(T));
  T *ck_s = reinterpret_cast<T *>(att_smem);
  T *cv_s = ck_s + kAttEntries * pk;
  float *q_s = reinterpret_cast<float *>(att_smem + att_stage_bytes(s, sizeof(T)));  // [G][rk]
  float *p_s = q_s + kAttMaxGroup * rk;                               // [G][64]
  float *ml_s = p_s + kAttMaxGroup * kAttEntries;                     // [G][4]
  float *acc_s = ml_s + 4 * kAttMaxGroup;                             // [G][rv]
  float *sw_s = acc_s + kAttMaxGroup * rv;                            // [G][kAttMaxSinks]
  float *f_s = sw_s + kAttMaxGroup * kAttMaxSinks;                    // [G][kAttMaxSplits]
  __shared__ int64_t rows_s[kAttEntries];
  __shared__ int last_flag;

  const int64_t L = valid_length(lengths[b], s.cache_rows);
  const int64_t n_top = smin<int64_t>(s.top_k, n_candidates(L, s.local_window));
  const int64_t n_win = smin<int64_t>(s.local_window, L);
  const int64_t n_sel = n_top + n_win;
  const int64_t e0 = (int64_t)split * kAttEntries;
  const int n_e = (int)smax<int64_t>(0, smin<int64_t>(kAttEntries, n_sel - e0));
  const int32_t *idx_b = idx + (int64_t)b * s.top_k;
  const T *ckb = coeff_k + (int64_t)b * s.cache_rows * rk;
  const T *cvb = coeff_v + (int64_t)b * s.cache_rows * rv;

  // 1. stage the split's rows; an entry outside [0, L) (which the top-k
  //    kernel never produces) is skipped with logit -inf.
  for (int e = threadIdx.x; e < kAttEntries; e += blockDim.x) {
    int64_t row = -1;
    if (e < n_e) {
      row = att_entry_row(idx_b, n_top, L, n_win, e0 + e, s.n_sink);
      if (row < 0 || row >= L) row = -1;
    }
    rows_s[e] = row;
  }
  __syncthreads();
  {
    const int ck_chunks = rk / V, cv_chunks = rv / V;
    for (int t = threadIdx.x; t < n_e * (ck_chunks + cv_chunks); t += blockDim.x) {
      const int e = t / (ck_chunks + cv_chunks), c = t - e * (ck_chunks + cv_chunks);
      const int64_t row = rows_s[e];
      if (row < 0) {  // keep skipped rows finite: their weights are zero
        T *dst = (c < ck_chunks) ? ck_s + e * pk + c * V : cv_s + e * pv + (c - ck_chunks) * V;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      if (c < ck_chunks)
        cp_async16(ck_s + e * pk + c * V, ckb + row * rk + c * V);
      else
        cp_async16(cv_s + e * pv + (c - ck_chunks) * V, cvb + row * rv + (c - ck_chunks) * V);
    }
  }
  for (int t = threadIdx.x; t < G * rk; t += blockDim.x) {
    const int j = t / rk, k = t - j * rk;
    q_s[j * rk + k] = qt_all[((int64_t)b * s.n_heads_q + g * G + j) * rk + k];
  }
  cp_async_wait_all();
  __syncthreads();

  // 2a. logits of (head j, entry e) pairs.
  for (int t = threadIdx.x; t < G * kAttEntries; t += blockDim.x) {
    const int j = t / kAttEntries, e = t - j * kAttEntries;
    float l = -INFINITY;
    if (e < n_e && rows_s[e] >= 0) l = dot_f32_store(q_s + j * rk, ck_s + e * pk, rk);
    p_s[j * kAttEntries + e] = l;
  }
  __syncthreads();
  // 2b. softmax partial per head: warp w takes head w.
  for (int j = wid; j < G; j += kAttThreads / 32) {
    const float l0 = p_s[j * kAttEntries + lane], l1 = p_s[j * kAttEntries + lane + 32];
    const float m = warp_max(fmaxf(l0, l1));
    const float p0 = (m == -INFINITY) ? 0.f : __expf(l0 - m);
    const float p1 = (m == -INFINITY) ? 0.f : __expf(l1 - m);
    const float l = warp_sum(p0 + p1);
    p_s[j * kAttEntries + lane] = p0;
    p_s[j * kAttEntries + lane + 32] = p1;
    if (lane == 0) {
      ml_s[j * 4] = m;
      ml_s[j * 4 + 1] = l;
    }
  }
  __syncthreads();
  // 2c. latent value sums, one column k per thread.
  for (int k = threadIdx.x; k < rv; k += blockDim.x) {
    float acc[kAttMaxGroup];
#pragma unroll
    for (int j = 0; j < kAttMaxGroup; ++j) acc[j] = 0.f;
    for (int e = 0; e < n_e; ++e) {
      const float v = to_f(cv_s[e * pv + k]);
#pragma unroll
      for (int j = 0; j < kAttMaxGroup; ++j)
        if (j < G) acc[j] = fmaf(p_s[j * kAttEntries + e], v, acc[j]);
    }
#pragma unroll
    for (int j = 0; j < kAttMaxGroup; ++j)
      if (j < G) part[(((int64_t)b * s.n_heads_q + g * G + j) * n_split + split) * (rv + 2) + 2 + k] = acc[j];
  }
  if (threadIdx.x < G) {
    float *pp = part + (((int64_t)b * s.n_heads_q + g * G + threadIdx.x) * n_split + split) * (rv + 2);
    pp[0] = ml_s[threadIdx.x * 4];
    pp[1] = ml_s[threadIdx.x * 4 + 1];
  }
  // 3. the last split CTA of this (problem, group) merges.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int t = atomicAdd(&tickets[(int64_t)b * s.n_heads_kv + g], 1u);
    last_flag = (t == (unsigned int)n_split - 1);
  }
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
  // Stage B^V[g] (d_h rows x rv) over the row buffers.
  T *bv_s = ck_s;
  const T *Bv = basis_v + (int64_t)b * Dp * rv + (int64_t)g * dh * rv;
  for (int t = threadIdx.x; t < dh * (rv / V); t += blockDim.x) {
    const int e = t / (rv / V), c = t - e * (rv / V);
    cp_async16(bv_s + e * pv + c * V, Bv + (int64_t)e * rv + c * V);
  }
  // Sink logits: one warp per (head, sink).
  const float qscale = rsqrtf((float)dh);
  for (int t = wid; t < G * ns; t += kAttThreads / 32) {
    const int j = t / ns, tk = t - j * ns;
    const T *qh = q + (((int64_t)b * s.query_window + s.query_window - 1) * s.n_heads_q + g * G + j) * dh;
    const T *kr = sink_k + ((int64_t)b * ns + tk) * Dp + (int64_t)g * dh;
    float d = 0.f;
    for (int e = lane; e < dh; e += 32) d = fmaf(to_f(qh[e]), to_f(kr[e]), d);
    d = warp_sum(d);
    if (lane == 0) sw_s[j * kAttMaxSinks + tk] = d * qscale;
  }
  __syncthreads();
  // Merge statistics per head (warp w takes head w): weights of the splits
  // f[j][sp] = exp(m_sp - M) / den and of the sinks, into shared memory.
  for (int j = wid; j < G; j += kAttThreads / 32) {
    const float *pb = part + ((int64_t)b * s.n_heads_q + g * G + j) * n_split * (rv + 2);
    float ms[kAttMaxSplits / 32], ls[kAttMaxSplits / 32];
    float M = -INFINITY;
#pragma unroll
    for (int u = 0; u < kAttMaxSplits / 32; ++u) {
      const int sp = lane + 32 * u;
      ms[u] = sp < n_split ? __ldcg(pb + sp * (rv + 2)) : -INFINITY;
      ls[u] = sp < n_split ? __ldcg(pb + sp * (rv + 2) + 1) : 0.f;
      M = fmaxf(M, ms[u]);
    }
    for (int tk = lane; tk < ns; tk += 32) M = fmaxf(M, sw_s[j * kAttMaxSinks + tk]);
    M = warp_max(M);
    float den = 0.f;
#pragma unroll
    for (int u = 0; u < kAttMaxSplits / 32; ++u) {
      ms[u] = (ms[u] == -INFINITY) ? 0.f : __expf(ms[u] - M);
      den += ls[u] * ms[u];
    }
    for (int tk = lane; tk < ns; tk += 32) den += __expf(sw_s[j * kAttMaxSinks + tk] - M);
    den = warp_sum(den);
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int u = 0; u < kAttMaxSplits / 32; ++u) {
      const int sp = lane + 32 * u;
      if (sp < n_split) f_s[j * kAttMaxSplits + sp] = ms[u] * inv;
    }
    __syncwarp();
    for (int tk = lane; tk < ns; tk += 32)
      sw_s[j * kAttMaxSinks + tk] = __expf(sw_s[j * kAttMaxSinks + tk] - M) * inv;
  }
  __syncthreads();
  // Latent accumulator per head: acc[j][k] = sum_split f[j][split] acc_split[k].
  // Each thread owns up to kOut outputs and reads their split values in
  // rounds of 4 splits, so kOut * 4 independent loads are in flight.
  {
    constexpr int kOut = 4;
    const int n_out = G * rv;
    for (int t0 = 0; t0 < n_out; t0 += kOut * kAttThreads) {
      const float *src[kOut];
      float a[kOut];
      int jj[kOut];
#pragma unroll
      for (int o = 0; o < kOut; ++o) {
        const int t = t0 + o * kAttThreads + threadIdx.x;
        const int j = (t < n_out) ? t / rv : 0, k = (t < n_out) ? t - j * rv : 0;
        jj[o] = j;
        src[o] = part + ((int64_t)b * s.n_heads_q + g * G + j) * n_split * (rv + 2) + 2 + k;
        a[o] = 0.f;
      }
      for (int sp = 0; sp < n_split; sp += 4) {
        float v[kOut][4];
#pragma unroll
        for (int o = 0; o < kOut; ++o)
#pragma unroll
          for (int u = 0; u < 4; ++u) v[o][u] = (sp + u < n_split) ? __ldcg(src[o] + (sp + u) * (rv + 2)) : 0.f;
#pragma unroll
        for (int o = 0; o < kOut; ++o)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (sp + u < n_split) a[o] = fmaf(f_s[jj[o] * kAttMaxSplits + sp + u], v[o][u], a[o]);
      }
#pragma unroll
      for (int o = 0; o < kOut; ++o) {
        const int t = t0 + o * kAttThreads + threadIdx.x;
        if (t < n_out) acc_s[t] = a[o];   // acc_s[j * rv + k] == acc_s[t]
      }
    }
  }
  cp_async_wait_all();
  __syncthreads();
  // out[h][e] = acc[j] . B^V[g*dh + e] + sum_t w_t sink_v[t][g*dh + e].
  for (int t = threadIdx.x; t < G * dh; t += blockDim.x) {
    const int j = t / dh, e = t - j * dh;
    float o = dot_f32_store(acc_s + j * rv, bv_s + e * pv, rv);
    for (int tk = 0; tk < ns; ++tk)
      o = fmaf(sw_s[j * kAttMaxSinks + tk], to_f(sink_v[((int64_t)b * ns + tk) * Dp + (int64_t)g * dh + e]), o);
    out[((int64_t)b * s.n_heads_q + g * G + j) * dh + e] = o;
  }
  if (threadIdx.x == 0) tickets[(int64_t)b * s.n_heads_kv + g] = 0u;
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
