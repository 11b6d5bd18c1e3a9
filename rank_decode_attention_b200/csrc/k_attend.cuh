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
//   0. before waiting for the top-k kernel, each CTA starts bulk copies of
//      the rows of B^V[g] its share of the output needs (an input);
//   1. CTA rank c takes an equal share of the selected rows, bulk-copies
//      their C_K / C_V rows into shared memory (all at once when they fit,
//      else in chunks), computes the logits of the G heads of group g, an
//      online softmax (running max, sum) and the latent value sums
//      acc[j][:] += p[j][e] c_V[e]; it also computes the sink logits of the
//      heads it will finish;
//   2. its partial (m, l, acc) stays in its shared memory.  After a cluster
//      barrier every CTA finishes its own slice of the output, (head j,
//      column e) pairs: it merges the ranks' partials of head j (read through
//      distributed shared memory) with the sink terms and maps the merged acc
//      through its staged rows of B^V[g].  A second cluster barrier keeps the
//      partials alive until every CTA is done.
#pragma once
#include "common.cuh"
#include "k_topk.cuh"
#include "umma.cuh"

namespace s4r {

constexpr int kAttThreads = 256;      // 8 warps
constexpr int kAttCluster = 8;        // CTAs per (kv group, problem)
constexpr int kAttEntriesMax = 256;   // selected rows staged at once per CTA
constexpr int kAttMaxGroup = 8;       // G <= 8
constexpr int kAttMaxSinks = 16;
constexpr size_t kAttSmemBudget = 224 * 1024;  // dynamic; leaves room for the static rows and barriers

// Row pitch (elements) of staged rows: 16-byte multiples whose 4-byte-word
// stride is 4 (mod 8), so the 16-byte reads of 8 consecutive rows fall in
// distinct bank quads.
__host__ __device__ inline int att_pitch(int n, int esize) {
  int words = (n * esize) / 4;
  while (words % 8 != 4) words += 4;
  return words * 4 / esize;
}

// Output items of a cluster rank: (head j, column e) pairs t = j*d_h + e in
// [t0, t1), needing rows e_lo .. e_hi-1 of B^V[g] (all d_h rows if the
// range spans two heads).
struct AttItems {
  int t0, t1, e_lo, e_hi;
};
__host__ __device__ inline AttItems att_items(int G, int dh, int n_ranks, int rank) {
  const int total = G * dh, per = (total + n_ranks - 1) / n_ranks;
  AttItems it;
  it.t0 = rank * per < total ? rank * per : total;
  it.t1 = it.t0 + per < total ? it.t0 + per : total;
  if (it.t1 <= it.t0) {
    it.e_lo = it.e_hi = 0;
  } else if (it.t0 / dh == (it.t1 - 1) / dh) {
    it.e_lo = it.t0 % dh;
    it.e_hi = (it.t1 - 1) % dh + 1;
  } else {
    it.e_lo = 0;
    it.e_hi = dh;
  }
  return it;
}

// Float counts of shared-memory regions are kept multiples of 4 (16 bytes),
// so every region starts 16-byte aligned.
__host__ __device__ inline size_t att_round4(size_t n) { return (n + 3) / 4 * 4; }

// Launch plan: CTAs per cluster, rows staged per pass (a multiple of 32) and
// B^V rows staged.
struct AttPlan {
  int n_ranks, e_cap, bv_rows;
};
__host__ __device__ inline size_t att_float_words(const Shape &s, int e_cap, int bv_rows) {
  return (size_t)kAttMaxGroup * s.rank_k          // q_s
         + (size_t)kAttMaxGroup * e_cap           // p_s: [entry][kAttMaxGroup]
         + att_round4((size_t)s.n_sink * bv_rows)  // sv_s: sink values of this CTA's output columns
         + (size_t)8 * att_pitch(s.rank_k, 2)     // qb_s: [16][pitch] bf16 split query (tensor-core B operand)
         + (size_t)kAttMaxGroup * 4               // ml_s: m, l, chunk scale
         + (size_t)kAttMaxGroup * (s.rank_v + 4)  // part_s: this CTA's (m, l, -, -, acc[rv]) per head
         + (size_t)2 * kAttCluster * (s.rank_v + 4)  // recv_s: every rank's partial of the <= 2 heads finished here
         + (size_t)2 * s.rank_v                   // acc_s: merged acc of those heads
         + (size_t)kAttMaxGroup * kAttMaxSinks    // sw_s: sink logits, then weights
         + (size_t)2 * kAttCluster                // f_s: merge weights of the ranks
         + (size_t)8 * att_pitch(e_cap, 2);       // pb_s: [16][pitch] bf16 split weights (tensor-core B operand)
}
__host__ __device__ inline size_t att_smem_bytes(const Shape &s, int esize, const AttPlan &pl) {
  const size_t rows = (size_t)pl.e_cap * (att_pitch(s.rank_k, esize) + att_pitch(s.rank_v, esize)) * esize;
  const size_t bv = (size_t)pl.bv_rows * att_pitch(s.rank_v, esize) * esize;
  return rows + bv + sizeof(float) * att_float_words(s, pl.e_cap, pl.bv_rows);
}
// CTAs per (kv group, problem): enough clusters to cover about two CTAs per
// SM, at most kAttCluster (a power of two), and at least G so that a CTA's
// output slice spans at most two heads (its receive buffers hold two).
__host__ inline int att_ranks(const Shape &s, int n_sms) {
  const int64_t units = (int64_t)s.n_heads_kv * s.batch;
  int lo = 1;
  while (lo < s.group) lo <<= 1;
  int n = kAttCluster;
  while (n > lo && units * n > 2 * (int64_t)n_sms) n >>= 1;
  return n;
}
__host__ inline AttPlan att_plan(const Shape &s, int esize, int n_ranks = kAttCluster) {
  AttPlan pl;
  pl.n_ranks = n_ranks;
  pl.bv_rows = 0;
  for (int c = 0; c < n_ranks; ++c) {
    const AttItems it = att_items(s.group, s.head_dim, n_ranks, c);
    pl.bv_rows = it.e_hi - it.e_lo > pl.bv_rows ? it.e_hi - it.e_lo : pl.bv_rows;
  }
  const int64_t per = ceil_div((int64_t)s.top_k + s.local_window, n_ranks);
  int e = (int)smin<int64_t>(kAttEntriesMax, smax<int64_t>(32, (per + 31) / 32 * 32));
  pl.e_cap = e;
  while (pl.e_cap > 32 && att_smem_bytes(s, esize, pl) > kAttSmemBudget) pl.e_cap -= 32;
  return pl;
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
__global__ void __launch_bounds__(kAttThreads, 1)
attend_kernel(Shape s, AttPlan pl, const int32_t *__restrict__ lengths, const int32_t *__restrict__ idx,
              const T *__restrict__ coeff_k, const T *__restrict__ coeff_v, const float *__restrict__ qt_all,
              const T *__restrict__ q, const T *__restrict__ basis_v, const T *__restrict__ sink_k,
              const T *__restrict__ sink_v, float *__restrict__ out, uint32_t *__restrict__ status) {
  extern __shared__ __align__(16) unsigned char att_smem[];
  constexpr int V = Vec16<T>::n;
  constexpr int kWarps = kAttThreads / 32;
  const int E = pl.e_cap;
  const int g = blockIdx.y, b = blockIdx.z;
  const uint32_t rank = cluster_ctarank();
  const int n_ranks = (int)gridDim.x;   // the launch makes gridDim.x CTAs one cluster
  const int G = s.group, rk = s.rank_k, rv = s.rank_v, dh = s.head_dim, Dp = s.d_model, ns = s.n_sink;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pk = att_pitch(rk, sizeof(T)), pv = att_pitch(rv, sizeof(T));
  T *ck_s = reinterpret_cast<T *>(att_smem);
  T *cv_s = ck_s + (size_t)E * pk;
  T *bv_s = cv_s + (size_t)E * pv;
  float *q_s = reinterpret_cast<float *>(bv_s + (size_t)pl.bv_rows * pv);  // [G][rk]
  float *p_s = q_s + kAttMaxGroup * rk;                     // [E][kAttMaxGroup] logits, then weights
  float *sv_s = p_s + kAttMaxGroup * E;                     // [ns][e_hi - e_lo] sink values
  bf16 *qb_s = reinterpret_cast<bf16 *>(sv_s + att_round4((size_t)ns * pl.bv_rows));  // [16][pq]
  const int pq = att_pitch(rk, 2);
  float *ml_s = reinterpret_cast<float *>(qb_s + 16 * pq);  // [G][4]
  const int pr = rv + 4;                                    // partial row: m, l, -, -, acc[rv]
  float *part_s = ml_s + kAttMaxGroup * 4;                  // [G][pr]
  float *recv_s = part_s + kAttMaxGroup * pr;               // [2][kAttCluster][pr]
  float *acc_s = recv_s + 2 * kAttCluster * pr;             // [2][rv]
  float *sw_s = acc_s + 2 * rv;                             // [G][kAttMaxSinks]
  float *f_s = sw_s + kAttMaxGroup * kAttMaxSinks;          // [2][kAttCluster]
  bf16 *pb_s = reinterpret_cast<bf16 *>(f_s + 2 * kAttCluster);  // [16][ppb]
  const int ppb = att_pitch(E, 2);
  __shared__ int64_t rows_s[kAttEntriesMax];
  __shared__ __align__(8) uint64_t stage_bar, bv_bar, recv_bar;

  // 0. This CTA's output items and their rows of B^V[g] (inputs: the copies
  // start before the wait for the top-k kernel).
  const AttItems it = att_items(G, dh, n_ranks, (int)rank);
  const T *Bv = basis_v + (int64_t)b * Dp * rv + (int64_t)g * dh * rv;
  const int j_lo = it.t1 > it.t0 ? it.t0 / dh : 0, j_hi = it.t1 > it.t0 ? (it.t1 - 1) / dh + 1 : 0;
  if (threadIdx.x == 0) {
    mbar_init(&stage_bar, 1);
    mbar_init(&bv_bar, 1);
    mbar_init(&recv_bar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&bv_bar, (uint32_t)((it.e_hi - it.e_lo) * rv * sizeof(T)));
    // Every rank's partial of each head finished here arrives by bulk copy.
    mbar_arrive_expect_tx(&recv_bar, (uint32_t)(n_ranks * (j_hi - j_lo) * pr * sizeof(float)));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < it.e_hi - it.e_lo; e += blockDim.x)
    bulk_load(bv_s + (size_t)e * pv, Bv + (int64_t)(it.e_lo + e) * rv, (uint32_t)(rv * sizeof(T)), &bv_bar);
  // The latent query (written by the projection kernel, which completed
  // before the top-k kernel started), the sink values of this CTA's output
  // columns and the sink logits of its heads: none of it depends on the
  // top-k kernel, so it is prepared while that kernel runs.
  for (int t = threadIdx.x; t < G * rk; t += blockDim.x) {
    const int j = t / rk, k = t - j * rk;
    q_s[j * rk + k] = __ldcg(qt_all + ((int64_t)b * s.n_heads_q + g * G + j) * rk + k);
  }
  // Tensor-core operand of the logits: column n = 2j + term holds head j's
  // latent query as two bf16 terms (hi, lo) whose sum keeps ~16 bits.
  for (int t = threadIdx.x; t < 16 * rk; t += blockDim.x) {
    const int n = t / rk, k = t - n * rk, j = n >> 1;
    float v = 0.f;
    if (j < G) {
      const float x = __ldcg(qt_all + ((int64_t)b * s.n_heads_q + g * G + j) * rk + k);
      const float hi = __bfloat162float(__float2bfloat16_rn(x));
      v = (n & 1) ? x - hi : hi;
    }
    qb_s[n * pq + k] = __float2bfloat16_rn(v);
  }
  for (int t = threadIdx.x; t < ns * (it.e_hi - it.e_lo); t += blockDim.x) {
    const int tk = t / (it.e_hi - it.e_lo), e = t - tk * (it.e_hi - it.e_lo);
    sv_s[t] = to_f(sink_v[((int64_t)b * ns + tk) * Dp + (int64_t)g * dh + it.e_lo + e]);
  }
  {
    const float qscale = rsqrtf((float)dh);
    const int nh = j_hi - j_lo;
    for (int t = wid; t < nh * ns; t += kWarps) {
      const int j = j_lo + t / ns, tk = t % ns;
      const T *qh = q + (((int64_t)b * s.query_window + s.query_window - 1) * s.n_heads_q + g * G + j) * dh;
      const T *kr = sink_k + ((int64_t)b * ns + tk) * Dp + (int64_t)g * dh;
      float d = 0.f;
      for (int e = lane; e < dh; e += 32) d = fmaf(to_f(qh[e]), to_f(kr[e]), d);
      d = warp_sum(d);
      if (lane == 0) sw_s[j * kAttMaxSinks + tk] = d * qscale;
    }
  }
  // Every rank's barriers are initialised before any rank copies into them.
  cluster_sync();
  pdl_wait();      // idx comes from the preceding kernel
  pdl_trigger();

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
  if (threadIdx.x < G) {
    ml_s[threadIdx.x * 4] = -INFINITY;   // running max
    ml_s[threadIdx.x * 4 + 1] = 0.f;     // running sum
  }
  float acc[kAttMaxGroup];
#pragma unroll
  for (int j = 0; j < kAttMaxGroup; ++j) acc[j] = 0.f;
  const int kcol = threadIdx.x;  // latent value column owned by this thread (< rv)
  // Tensor-core path of the latent value sums (bf16 storage): acc^T[k][n] =
  // sum_e C_V[e][k] W[e][n], W column n = 2j + term holding head j's
  // weights as two bf16 terms; warp w owns the 16-column tiles w, w + 8.
  const bool tc_acc = sizeof(T) == 2 && rv % 16 == 0;
  const int n_nt = (2 * G + 7) / 8;
  float accf[2][2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int d = 0; d < 4; ++d) accf[a][c][d] = 0.f;

  uint32_t phase = 0;
  bool staged_ok = true;   // false once a wait for staged rows gave up: no further chunks are staged
  for (int64_t c0 = e_begin; c0 < e_end && staged_ok; c0 += E) {
    const int n_e = (int)smin<int64_t>(E, e_end - c0);
    __syncthreads();  // previous chunk fully consumed
    int live = 0;     // E <= blockDim.x: at most one entry per thread
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int64_t row = -1;
      if (e < n_e) {
        row = att_entry_row(idx_b, n_top, L, n_win, c0 + e, s.n_sink);
        if (row < 0 || row >= L) row = -1;  // never produced by the top-k kernel
      }
      rows_s[e] = row;
      live = row >= 0;
    }
    // One bulk copy per row and operand (rows are 16-byte multiples), all
    // completing on stage_bar; skipped rows are zeroed by plain stores.
    const int n_live = __syncthreads_count(live);
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&stage_bar, (uint32_t)(n_live * (rk + rv) * sizeof(T)));
    __syncthreads();
    for (int t = threadIdx.x; t < 2 * E; t += blockDim.x) {
      const int e = t % E;
      const bool is_v = t >= E;
      const int64_t row = e < n_e ? rows_s[e] : -1;
      T *dst = is_v ? cv_s + (size_t)e * pv : ck_s + (size_t)e * pk;
      const int n = is_v ? rv : rk;
      if (row >= 0) {
        bulk_load(dst, is_v ? cvb + row * rv : ckb + row * rk, (uint32_t)(n * sizeof(T)), &stage_bar);
      } else {
        for (int c = 0; c < n; c += V) *reinterpret_cast<uint4 *>(dst + c) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // Every thread waits (bounded) and sees the same outcome unless the copies
    // land right at the limit; the vote makes the decision uniform.
    staged_ok = __syncthreads_and(mbar_wait(&stage_bar, phase, status)) != 0;
    phase ^= 1u;
    if (sizeof(T) == 2 && rk % 16 == 0) {
      // logits on the tensor cores: per warp, 16-entry tiles of
      // C_K[16 x rk] . Qsplit[rk x 8] (mma m16n8k16, bf16 in, fp32 out); the
      // accumulator of row e, column 2j + term is split over lanes
      // (g = lane / 4 rows, t = lane % 4 column pairs).
      const int gq = lane >> 2, tq = lane & 3;
      const int n_nt = (2 * G + 7) / 8;
      for (int mt = wid; mt < E / 16; mt += kWarps) {
        const int e0 = mt * 16 + gq, e1 = e0 + 8;
        const uint32_t *a_lo = reinterpret_cast<const uint32_t *>(ck_s + (size_t)e0 * pk) + tq;
        const uint32_t *a_hi = reinterpret_cast<const uint32_t *>(ck_s + (size_t)e1 * pk) + tq;
        const bool ok0 = e0 < n_e && rows_s[e0] >= 0, ok1 = e1 < n_e && rows_s[e1] >= 0;
        for (int nt = 0; nt < n_nt; ++nt) {
          const uint32_t *bq = reinterpret_cast<const uint32_t *>(qb_s + (size_t)(nt * 8 + gq) * pq) + tq;
          float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll 4
          for (int ks = 0; ks < rk / 16; ++ks) {
            const uint32_t a0 = a_lo[ks * 8], a1 = a_hi[ks * 8], a2 = a_lo[ks * 8 + 4], a3 = a_hi[ks * 8 + 4];
            const uint32_t b0 = bq[ks * 8], b1 = bq[ks * 8 + 4];
            asm volatile(
                "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                "{%0,%1,%2,%3};"
                : "+f"(c0), "+f"(c1), "+f"(c2), "+f"(c3)
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
          }
          const int j = nt * 4 + tq;   // columns 2j, 2j + 1: the two terms of head j
          if (j < G) {
            p_s[e0 * kAttMaxGroup + j] = ok0 ? c0 + c1 : -INFINITY;
            p_s[e1 * kAttMaxGroup + j] = ok1 ? c2 + c3 : -INFINITY;
          }
        }
      }
    } else
    // logits: the thread of entry e computes all G heads, reading its key
    // row once and the latent queries as broadcast float4s
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      float l0[kAttMaxGroup], l1[kAttMaxGroup];
#pragma unroll
      for (int j = 0; j < kAttMaxGroup; ++j) l0[j] = l1[j] = 0.f;
      const bool ok = e < n_e && rows_s[e] >= 0;
      if (ok) {
        const T *kr = ck_s + (size_t)e * pk;
        for (int k = 0; k < rk; k += V) {
          float xv[V];
          load16(kr + k, xv);
#pragma unroll
          for (int j = 0; j < kAttMaxGroup; ++j) {
            if (j < G) {
#pragma unroll
              for (int u = 0; u < V; u += 4) {
                const float4 qv = *reinterpret_cast<const float4 *>(q_s + j * rk + k + u);
                l0[j] = fmaf(qv.x, xv[u], l0[j]);
                l1[j] = fmaf(qv.y, xv[u + 1], l1[j]);
                l0[j] = fmaf(qv.z, xv[u + 2], l0[j]);
                l1[j] = fmaf(qv.w, xv[u + 3], l1[j]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kAttMaxGroup; ++j)
        if (j < G) p_s[e * kAttMaxGroup + j] = ok ? l0[j] + l1[j] : -INFINITY;
    }
    __syncthreads();
    // online softmax update per head (warp j), E / 32 entries per lane
    for (int j = wid; j < G; j += kWarps) {
      constexpr int kPerMax = kAttEntriesMax / 32;
      const int n_per = E / 32;
      float lv[kPerMax];
      float mc = -INFINITY;
#pragma unroll
      for (int u = 0; u < kPerMax; ++u) {
        lv[u] = u < n_per ? p_s[(lane + 32 * u) * kAttMaxGroup + j] : -INFINITY;
        mc = fmaxf(mc, lv[u]);
      }
      const float m_old = ml_s[j * 4];
      const float m_new = fmaxf(m_old, warp_max(mc));
      float csum = 0.f;
#pragma unroll
      for (int u = 0; u < kPerMax; ++u) {
        if (u < n_per) {
          const float pu = (m_new == -INFINITY) ? 0.f : __expf(lv[u] - m_new);
          p_s[(lane + 32 * u) * kAttMaxGroup + j] = pu;
          csum += pu;
        }
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
    if (tc_acc) {
      // Split weights into the B operand (the 8 n_nt columns the products
      // read), then one m16n8k16 per (tile, 16 entries).
      for (int t = threadIdx.x; t < 8 * n_nt * E; t += blockDim.x) {
        const int n = t / E, e = t - n * E, j = n >> 1;
        const float pv_ = j < G ? p_s[e * kAttMaxGroup + j] : 0.f;
        const float hi = __bfloat162float(__float2bfloat16_rn(pv_));
        pb_s[n * ppb + e] = __float2bfloat16_rn((n & 1) ? pv_ - hi : hi);
      }
      __syncthreads();
      const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int mt = wid + a * kWarps;
        if (mt < rv / 16) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int j = c * 4 + tq;
            const float sc = (c < n_nt && j < G) ? ml_s[j * 4 + 2] : 0.f;
#pragma unroll
            for (int d = 0; d < 4; ++d) accf[a][c][d] *= sc;
          }
          for (int ks = 0; ks < E / 16; ++ks) {
            // A = C_V^T tile: four 8x8 blocks (entries x columns) loaded transposed.
            const int m = lane >> 3;
            const int e = ks * 16 + ((m & 2) ? 8 : 0) + (lane & 7);
            const int c0 = mt * 16 + ((m & 1) ? 8 : 0);
            uint32_t a0, a1, a2, a3;
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                         : "r"(smem_u32(cv_s + (size_t)e * pv + c0)));
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (c < n_nt) {
                const uint32_t *bw = reinterpret_cast<const uint32_t *>(pb_s + (size_t)(c * 8 + gq) * ppb + ks * 16) + tq;
                const uint32_t b0 = bw[0], b1 = bw[4];
                asm volatile(
                    "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                    "{%0,%1,%2,%3};"
                    : "+f"(accf[a][c][0]), "+f"(accf[a][c][1]), "+f"(accf[a][c][2]), "+f"(accf[a][c][3])
                    : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
              }
            }
          }
        }
      }
    } else if (kcol < rv) {
      float sc[kAttMaxGroup];
#pragma unroll
      for (int j = 0; j < kAttMaxGroup; ++j) {
        sc[j] = (j < G) ? ml_s[j * 4 + 2] : 0.f;
        acc[j] *= sc[j];
      }
#pragma unroll 4
      for (int e = 0; e < n_e; ++e) {
        const float v = to_f(cv_s[(size_t)e * pv + kcol]);
        const float4 pa = *reinterpret_cast<const float4 *>(p_s + e * kAttMaxGroup);
        acc[0] = fmaf(pa.x, v, acc[0]);
        acc[1] = fmaf(pa.y, v, acc[1]);
        acc[2] = fmaf(pa.z, v, acc[2]);
        acc[3] = fmaf(pa.w, v, acc[3]);
        if (G > 4) {
          const float4 pb = *reinterpret_cast<const float4 *>(p_s + e * kAttMaxGroup + 4);
          acc[4] = fmaf(pb.x, v, acc[4]);
          acc[5] = fmaf(pb.y, v, acc[5]);
          acc[6] = fmaf(pb.z, v, acc[6]);
          acc[7] = fmaf(pb.w, v, acc[7]);
        }
      }
    }
  }
  // This CTA's partial (m, l, acc) of every head, then stored into the CTAs
  // that finish each head.
  if (tc_acc) {
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int mt = wid + a * kWarps;
      if (mt < rv / 16) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int j = c * 4 + tq;
          if (c < n_nt && j < G) {
            part_s[j * pr + 4 + mt * 16 + gq] = accf[a][c][0] + accf[a][c][1];
            part_s[j * pr + 4 + mt * 16 + gq + 8] = accf[a][c][2] + accf[a][c][3];
          }
        }
      }
    }
  } else if (kcol < rv) {
#pragma unroll
    for (int j = 0; j < kAttMaxGroup; ++j)
      if (j < G) part_s[j * pr + 4 + kcol] = acc[j];
  }
  if (threadIdx.x < G) {
    part_s[threadIdx.x * pr] = ml_s[threadIdx.x * 4];
    part_s[threadIdx.x * pr + 1] = ml_s[threadIdx.x * 4 + 1];
  }
  // Bulk copies (the async proxy) read what the threads just wrote.
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  // One copy per (rank finishing head j, head j) of this CTA's partial row.
  if (threadIdx.x < n_ranks * 2) {
    const int r2 = threadIdx.x >> 1, jj = threadIdx.x & 1;
    const AttItems it2 = att_items(G, dh, n_ranks, r2);
    if (it2.t1 > it2.t0) {
      const int jlo2 = it2.t0 / dh, nh2 = (it2.t1 - 1) / dh + 1 - jlo2;
      if (jj < nh2)
        bulk_copy_to_peer(cluster_map(recv_s + ((size_t)jj * kAttCluster + rank) * pr, (uint32_t)r2),
                          part_s + (size_t)(jlo2 + jj) * pr, (uint32_t)(pr * sizeof(float)),
                          cluster_map(&recv_bar, (uint32_t)r2));
    }
  }
  mbar_wait(&recv_bar, 0, status);    // every partial of the heads finished here has arrived
  // Every copy into this CTA is done.  A sender learns that its own copies
  // have been read only from the receivers, so no CTA leaves before all have
  // arrived here (the wait is at the end, after the merge and the output).
  // The arrive publishes no data, hence relaxed.
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // Merge weights of the heads this CTA finishes (warp per head; ranks = lanes).
  for (int jj = wid; jj < j_hi - j_lo; jj += kWarps) {
    const int j = j_lo + jj;
    float mr = -INFINITY, lr = 0.f;
    if (lane < n_ranks) {
      mr = recv_s[((size_t)jj * kAttCluster + lane) * pr];
      lr = recv_s[((size_t)jj * kAttCluster + lane) * pr + 1];
    }
    float M = mr;
    for (int tk = lane; tk < ns; tk += 32) M = fmaxf(M, sw_s[j * kAttMaxSinks + tk]);
    M = warp_max(M);
    const float fr = (mr == -INFINITY) ? 0.f : __expf(mr - M);
    float den = lr * fr;
    for (int tk = lane; tk < ns; tk += 32) den += __expf(sw_s[j * kAttMaxSinks + tk] - M);
    den = warp_sum(den);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    if (lane < n_ranks) f_s[jj * kAttCluster + lane] = fr * inv;
    __syncwarp();
    for (int tk = lane; tk < ns; tk += 32)
      sw_s[j * kAttMaxSinks + tk] = __expf(sw_s[j * kAttMaxSinks + tk] - M) * inv;
  }
  __syncthreads();
  // acc[j][k] = sum_r f[j][r] acc_r[j][k]
  for (int t = threadIdx.x; t < (j_hi - j_lo) * rv; t += blockDim.x) {
    const int jj = t / rv, k = t % rv;
    float a = 0.f;
#pragma unroll
    for (int r = 0; r < kAttCluster; ++r)
      if (r < n_ranks) a = fmaf(f_s[jj * kAttCluster + r], recv_s[((size_t)jj * kAttCluster + r) * pr + 4 + k], a);
    acc_s[jj * rv + k] = a;
  }
  mbar_wait(&bv_bar, 0, status);
  __syncthreads();
  // out[h][e] = acc[j] . B^V[g*dh + e] + sum_t w_t sink_v[t][g*dh + e], four
  // threads per output (16-byte chunks c = part, part + 4, ...).
  const int n_items = it.t1 - it.t0;
  for (int base = 0; base < 4 * n_items; base += blockDim.x) {
    const int t = base + (int)threadIdx.x, item = t >> 2, part = t & 3;
    const bool act = t < 4 * n_items;
    float o = 0.f;
    int j = 0, e = 0;
    if (act) {
      j = (it.t0 + item) / dh;
      e = (it.t0 + item) - j * dh;
      const float *av = acc_s + (j - j_lo) * rv;
      const T *br = bv_s + (size_t)(e - it.e_lo) * pv;
      for (int c = part * V; c < rv; c += 4 * V) {
        float xv[V];
        load16(br + c, xv);
#pragma unroll
        for (int u = 0; u < V; ++u) o = fmaf(av[c + u], xv[u], o);
      }
    }
    o += __shfl_xor_sync(0xffffffffu, o, 1);
    o += __shfl_xor_sync(0xffffffffu, o, 2);
    if (act && part == 0) {
      for (int tk = 0; tk < ns; ++tk)
        o = fmaf(sw_s[j * kAttMaxSinks + tk], sv_s[tk * (it.e_hi - it.e_lo) + (e - it.e_lo)], o);
      out[((int64_t)b * s.n_heads_q + g * G + j) * dh + e] = o;
    }
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
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
