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
// One launch; the kAttCluster CTAs of a (kv group g, problem) form a thread
// block cluster, 256 threads each:
//   1. CTA rank c takes an equal share of the selected rows and walks it in
//      chunks of 128 rows (64 for fp32 storage): cp.async the chunk's C_K / C_V rows, logits of the G
//      heads of group g, online softmax (running max, sum) and the latent
//      value sums acc[j][:] += p[j][e] c_V[e];
//   2. its partial (m, l, acc) stays in its shared memory; after a cluster
//      barrier rank 0 reads the other ranks' partials through distributed
//      shared memory, merges them with the sink logits, maps acc through
//      B^V[g] and writes out; a second cluster barrier keeps the partials
//      alive until rank 0 is done.
#pragma once
#include "common.cuh"
#include "k_topk.cuh"
#include "umma.cuh"

namespace s4r {

constexpr int kAttThreads = 256;      // 8 warps
constexpr int kAttCluster = 8;        // CTAs per (kv group, problem)
constexpr int kAttEntriesMax = 128;   // selected rows per chunk (bf16 storage; 64 for fp32)
template <typename T> __host__ __device__ constexpr int att_entries() { return sizeof(T) == 2 ? 128 : 64; }
constexpr int kAttMaxGroup = 8;       // G <= 8
constexpr int kAttMaxSinks = 16;      // sinks merged by rank 0

// Row pitch (elements) of staged rows: 16-byte multiples whose 4-byte-word
// stride is 4 (mod 8), so the 16-byte reads of 8 consecutive rows fall in
// distinct bank quads.
__host__ __device__ inline int att_pitch(int n, int esize) {
  int words = (n * esize) / 4;
  while (words % 8 != 4) words += 4;
  return words * 4 / esize;
}
__host__ __device__ inline size_t att_stage_bytes(const Shape &s, int esize) {
  const size_t rows = (size_t)(esize == 2 ? 128 : 64) * (att_pitch(s.rank_k, esize) + att_pitch(s.rank_v, esize)) * esize;
  const size_t bv = (size_t)s.head_dim * att_pitch(s.rank_v, esize) * esize;
  return rows > bv ? rows : bv;
}
__host__ __device__ inline size_t att_float_words(const Shape &s) {
  return (size_t)kAttMaxGroup * s.rank_k          // q_s
         + (size_t)kAttMaxGroup * kAttEntriesMax  // p_s
         + (size_t)kAttMaxGroup * 4               // ml_s: m, l, chunk scale, merged inverse
         + (size_t)kAttMaxGroup * (s.rank_v + 2)  // part_s: this CTA's m, l, acc[rv] per head
         + (size_t)kAttMaxGroup * s.rank_v        // acc_s (rank 0)
         + (size_t)kAttMaxGroup * kAttMaxSinks    // sw_s
         + (size_t)kAttMaxGroup * kAttCluster;    // f_s: merge weights of the ranks
}
__host__ inline size_t att_smem_bytes(const Shape &s, int esize) {
  return att_stage_bytes(s, esize) + sizeof(float) * att_float_words(s);
}

// Row number of selected entry e (top-k list first, then the window).
__device__ __forceinline__ int64_t att_entry_row(const int32_t *idx_b, int64_t n_top, int64_t L,
                                                 int64_t n_win, int64_t e, int32_t n_sink) {
  if (e < n_top) return (int64_t)idx_b[e] - n_sink;
  return L - n_win + (e - n_top);
}

// Dot product of n (a multiple of 8) fp32 values with n storage values,
// 16-byte reads, four independent partial sums.
template <typename T>
__device__ __forceinline__ float dot_f32_store(const float *a, const T *x, int n) {
  constexpr int V = Vec16<T>::n;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = 0; k < n; k += V) {
    float xv[V];
    load16(x + k, xv);
#pragma unroll
    for (int u = 0; u < V; ++u) acc[u & 3] = fmaf(a[k + u], xv[u], acc[u & 3]);
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

template <typename T>
__global__ void __launch_bounds__(kAttThreads)
attend_kernel(Shape s, const int32_t *__restrict__ lengths, const int32_t *__restrict__ idx,
              const T *__restrict__ coeff_k, const T *__restrict__ coeff_v, const float *__restrict__ qt_all,
              const T *__restrict__ q, const T *__restrict__ basis_v, const T *__restrict__ sink_k,
              const T *__restrict__ sink_v, float *__restrict__ out) {
  extern __shared__ __align__(16) unsigned char att_smem[];
  constexpr int V = Vec16<T>::n;
  constexpr int kWarps = kAttThreads / 32;
  constexpr int kAttEntries = att_entries<T>();
  const int g = blockIdx.y, b = blockIdx.z;
  const uint32_t rank = cluster_ctarank();
  const int n_ranks = (int)gridDim.x;   // the launch makes gridDim.x CTAs one cluster
  const int G = s.group, rk = s.rank_k, rv = s.rank_v, dh = s.head_dim, Dp = s.d_model, ns = s.n_sink;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int pk = att_pitch(rk, sizeof(T)), pv = att_pitch(rv, sizeof(T));
  T *ck_s = reinterpret_cast<T *>(att_smem);
  T *cv_s = ck_s + kAttEntries * pk;
  float *q_s = reinterpret_cast<float *>(att_smem + att_stage_bytes(s, sizeof(T)));  // [G][rk]
  float *p_s = q_s + kAttMaxGroup * rk;                     // [G][entries] logits, then weights
  float *ml_s = p_s + kAttMaxGroup * kAttEntries;           // [G][4]
  float *part_s = ml_s + kAttMaxGroup * 4;                  // [G][rv + 2]
  float *acc_s = part_s + kAttMaxGroup * (rv + 2);          // [G][rv]
  float *sw_s = acc_s + kAttMaxGroup * rv;                  // [G][kAttMaxSinks]
  float *f_s = sw_s + kAttMaxGroup * kAttMaxSinks;          // [G][kAttCluster]
  __shared__ int64_t rows_s[kAttEntriesMax];
  __shared__ __align__(8) uint64_t stage_bar;

  const int64_t L = valid_length(lengths[b], s.cache_rows);
  const int64_t n_top = smin<int64_t>(s.top_k, n_candidates(L, s.local_window));
  const int64_t n_win = smin<int64_t>(s.local_window, L);
  const int64_t n_sel = n_top + n_win;
  const int64_t per = ceil_div(n_sel, n_ranks);
  const int64_t e_begin = smin<int64_t>(n_sel, (int64_t)rank * per);
  const int64_t e_end = smin<int64_t>(n_sel, e_begin + per);
  const int32_t *idx_b = idx + (int64_t)b * s.top_k;
  const T *ckb = coeff_k + (int64_t)b * s.cache_rows * rk;
  const T *cvb = coeff_v + (int64_t)b * s.cache_rows * rv;

  for (int t = threadIdx.x; t < G * rk; t += blockDim.x) {
    const int j = t / rk, k = t - j * rk;
    q_s[j * rk + k] = qt_all[((int64_t)b * s.n_heads_q + g * G + j) * rk + k];
  }
  if (threadIdx.x == 0) {
    mbar_init(&stage_bar, 1);
    mbar_fence_init();
  }
  if (threadIdx.x < G) {
    ml_s[threadIdx.x * 4] = -INFINITY;   // running max
    ml_s[threadIdx.x * 4 + 1] = 0.f;     // running sum
  }
  float acc[kAttMaxGroup];
#pragma unroll
  for (int j = 0; j < kAttMaxGroup; ++j) acc[j] = 0.f;
  const int kcol = threadIdx.x;  // latent value column owned by this thread (< rv)

  uint32_t phase = 0;
  for (int64_t c0 = e_begin; c0 < e_end; c0 += kAttEntries) {
    const int n_e = (int)smin<int64_t>(kAttEntries, e_end - c0);
    __syncthreads();  // previous chunk fully consumed
    for (int e = threadIdx.x; e < kAttEntries; e += blockDim.x) {
      int64_t row = -1;
      if (e < n_e) {
        row = att_entry_row(idx_b, n_top, L, n_win, c0 + e, s.n_sink);
        if (row < 0 || row >= L) row = -1;  // never produced by the top-k kernel
      }
      rows_s[e] = row;
    }
    __syncthreads();
    // One bulk copy per row and operand (rows are 16-byte multiples), all
    // completing on stage_bar; skipped rows are zeroed by plain stores.
    if (threadIdx.x == 0) {
      uint32_t bytes = 0;
      for (int e = 0; e < n_e; ++e)
        if (rows_s[e] >= 0) bytes += (uint32_t)((rk + rv) * sizeof(T));
      mbar_arrive_expect_tx(&stage_bar, bytes);
    }
    __syncthreads();
    if (threadIdx.x < 2 * n_e) {
      const int e = threadIdx.x % n_e;
      const bool is_v = threadIdx.x >= n_e;
      const int64_t row = rows_s[e];
      T *dst = is_v ? cv_s + e * pv : ck_s + e * pk;
      const int n = is_v ? rv : rk;
      if (row >= 0) {
        bulk_load(dst, is_v ? cvb + row * rv : ckb + row * rk, (uint32_t)(n * sizeof(T)), &stage_bar);
      } else {
        for (int c = 0; c < n; c += V) *reinterpret_cast<uint4 *>(dst + c) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    mbar_wait(&stage_bar, phase, nullptr);
    phase ^= 1u;
    __syncthreads();
    // logits of (head j, entry e) pairs
    for (int t = threadIdx.x; t < G * kAttEntries; t += blockDim.x) {
      const int j = t / kAttEntries, e = t - j * kAttEntries;
      float l = -INFINITY;
      if (e < n_e && rows_s[e] >= 0) l = dot_f32_store(q_s + j * rk, ck_s + e * pk, rk);
      p_s[j * kAttEntries + e] = l;
    }
    __syncthreads();
    // online softmax update per head (warp j), kAttEntries / 32 entries per lane
    for (int j = wid; j < G; j += kWarps) {
      constexpr int kPer = kAttEntries / 32;
      float lv[kPer];
      float mc = -INFINITY;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        lv[u] = p_s[j * kAttEntries + lane + 32 * u];
        mc = fmaxf(mc, lv[u]);
      }
      const float m_old = ml_s[j * 4];
      const float m_new = fmaxf(m_old, warp_max(mc));
      float csum = 0.f;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const float pu = (m_new == -INFINITY) ? 0.f : __expf(lv[u] - m_new);
        p_s[j * kAttEntries + lane + 32 * u] = pu;
        csum += pu;
      }
      csum = warp_sum(csum);
      if (lane == 0) {
        const float scale = (m_old == -INFINITY) ? 0.f : __expf(m_old - m_new);
        ml_s[j * 4] = m_new;
        ml_s[j * 4 + 1] = ml_s[j * 4 + 1] * scale + csum;
        ml_s[j * 4 + 2] = scale;
      }
    }
    __syncthreads();
    if (kcol < rv) {
      float sc[kAttMaxGroup];
#pragma unroll
      for (int j = 0; j < kAttMaxGroup; ++j) {
        sc[j] = (j < G) ? ml_s[j * 4 + 2] : 0.f;
        acc[j] *= sc[j];
      }
      for (int e = 0; e < n_e; ++e) {
        const float v = to_f(cv_s[e * pv + kcol]);
#pragma unroll
        for (int j = 0; j < kAttMaxGroup; ++j)
          if (j < G) acc[j] = fmaf(p_s[j * kAttEntries + e], v, acc[j]);
      }
    }
  }
  // This CTA's partial, kept in shared memory for rank 0.
  if (kcol < rv)
#pragma unroll
    for (int j = 0; j < kAttMaxGroup; ++j)
      if (j < G) part_s[j * (rv + 2) + 2 + kcol] = acc[j];
  __syncthreads();
  if (threadIdx.x < G) {
    part_s[threadIdx.x * (rv + 2)] = ml_s[threadIdx.x * 4];
    part_s[threadIdx.x * (rv + 2) + 1] = ml_s[threadIdx.x * 4 + 1];
  }
  T *bv_s = ck_s;
  const T *Bv = basis_v + (int64_t)b * Dp * rv + (int64_t)g * dh * rv;
  if (rank == 0) {
    // Stage B^V[g] (d_h rows x rv) over the row buffers while the cluster syncs.
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&stage_bar, (uint32_t)(dh * rv * sizeof(T)));
    __syncthreads();
    for (int e = threadIdx.x; e < dh; e += blockDim.x)
      bulk_load(bv_s + e * pv, Bv + (int64_t)e * rv, (uint32_t)(rv * sizeof(T)), &stage_bar);
  }
  cluster_sync();  // every partial is in place
  if (rank == 0) {
    // Sink logits: one warp per (head, sink).
    const float qscale = rsqrtf((float)dh);
    for (int t = wid; t < G * ns; t += kWarps) {
      const int j = t / ns, tk = t - j * ns;
      const T *qh = q + (((int64_t)b * s.query_window + s.query_window - 1) * s.n_heads_q + g * G + j) * dh;
      const T *kr = sink_k + ((int64_t)b * ns + tk) * Dp + (int64_t)g * dh;
      float d = 0.f;
      for (int e = lane; e < dh; e += 32) d = fmaf(to_f(qh[e]), to_f(kr[e]), d);
      d = warp_sum(d);
      if (lane == 0) sw_s[j * kAttMaxSinks + tk] = d * qscale;
    }
    __syncthreads();
    // Merge weights per head (warp j): ranks r = lanes 0 .. n_ranks-1.
    for (int j = wid; j < G; j += kWarps) {
      float mr = -INFINITY, lr = 0.f;
      if (lane < n_ranks) {
        const uint32_t base = cluster_map(part_s + j * (rv + 2), (uint32_t)lane);
        mr = ld_cluster_f32(base);
        lr = ld_cluster_f32(base + 4);
      }
      float M = mr;
      for (int tk = lane; tk < ns; tk += 32) M = fmaxf(M, sw_s[j * kAttMaxSinks + tk]);
      M = warp_max(M);
      const float fr = (mr == -INFINITY) ? 0.f : __expf(mr - M);
      float den = lr * fr;
      for (int tk = lane; tk < ns; tk += 32) den += __expf(sw_s[j * kAttMaxSinks + tk] - M);
      den = warp_sum(den);
      const float inv = den > 0.f ? 1.f / den : 0.f;
      if (lane < n_ranks) f_s[j * kAttCluster + lane] = fr * inv;
      __syncwarp();
      for (int tk = lane; tk < ns; tk += 32)
        sw_s[j * kAttMaxSinks + tk] = __expf(sw_s[j * kAttMaxSinks + tk] - M) * inv;
    }
    __syncthreads();
    // acc[j][k] = sum_r f[j][r] acc_r[j][k], read through distributed shared memory.
    for (int t = threadIdx.x; t < G * rv; t += blockDim.x) {
      const int j = t / rv, k = t - j * rv;
      float v[kAttCluster];
#pragma unroll
      for (int r = 0; r < kAttCluster; ++r)
        v[r] = (r < n_ranks) ? ld_cluster_f32(cluster_map(part_s + j * (rv + 2) + 2 + k, (uint32_t)r)) : 0.f;
      float a = 0.f;
#pragma unroll
      for (int r = 0; r < kAttCluster; ++r)
        if (r < n_ranks) a = fmaf(f_s[j * kAttCluster + r], v[r], a);
      acc_s[t] = a;
    }
    mbar_wait(&stage_bar, phase, nullptr);
    __syncthreads();
    // out[h][e] = acc[j] . B^V[g*dh + e] + sum_t w_t sink_v[t][g*dh + e].
    for (int t = threadIdx.x; t < G * dh; t += blockDim.x) {
      const int j = t / dh, e = t - j * dh;
      float o = dot_f32_store(acc_s + j * rv, bv_s + e * pv, rv);
      for (int tk = 0; tk < ns; ++tk)
        o = fmaf(sw_s[j * kAttMaxSinks + tk], to_f(sink_v[((int64_t)b * ns + tk) * Dp + (int64_t)g * dh + e]), o);
      out[((int64_t)b * s.n_heads_q + g * G + j) * dh + e] = o;
    }
  }
  cluster_sync();  // rank 0 has read every partial
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
