// k_attend_rows.cuh -- sparse reconstruction + exact attention with the
// selected rows split over a thread-block cluster and every head in every CTA
// (bf16 storage).
//
// The mathematics is that of k_attend.cuh: Eqs. 16-18 of S4R (review page,
// "Core claim"; "assumptions": sinks stay in full precision), evaluated in
// absorbed form,
//   q_h . k_hat_i = (q_h B^K[g]) . c_K,i = qt_h . c_K,i
//   sum_i p_hi v_hat_i[g] = (sum_i p_hi c_V,i) B^V[g]^T,
// where qt_h is the projection kernel's latent query of head h (already
// scaled by 1/sqrt(d_h)) and B[g] are the d_h rows of a basis that belong to
// kv group g = h / G.
//
// The selected rows (top-k list, then the local window) are the same for
// every kv group, so each is read once: the NC CTAs of a problem's cluster
// take contiguous shares of the selection list.  CTA c
//   0. before waiting for the top-k kernel, starts 16-byte asynchronous
//      copies of the rows of B^V for the heads it will finish, splits every
//      head's latent query into two bf16 terms (hi + lo, ~16 mantissa bits)
//      and forms the sink logits of its heads;
//   1. per chunk of at most 128 rows: copies their C_K rows, then their C_V
//      rows (16-byte asynchronous copies; the C_V copies are still in flight
//      while the logits are formed), and computes for all H_q heads at once
//      (two warps per 16-row tile of logits, one warp per 16 latent columns
//      of the value sums)
//        logits[row][h] = C_K . Qt^T                 (mma.sync m16n8k16)
//        p = exp(logit - m_h) with a running max m_h and sum l_h per head
//        acc^T[k][h] = acc^T * rescale + C_V^T . p   (mma.sync m16n8k16)
//      with p split into two bf16 terms like the query; C_K and C_V are exact
//      in bf16, and every product is accumulated in fp32;
//   2. leaves its partial (m_h, l_h, acc_h) of every head in its shared
//      memory; after one cluster barrier it finishes heads
//      c*H_q/NC .. (c+1)*H_q/NC - 1: merges the NC partials of each (read
//      through distributed shared memory) with the head's sink terms and maps
//      the merged acc through the staged rows of B^V[g].
// The contractions are a few MFLOP per call: the kernel is bound by the
// latency of the row copies and the merge, not by the tensor pipe.
#pragma once
#include "common.cuh"
#include "k_attend.cuh"
#include "umma.cuh"

namespace s4r {

constexpr int kArThreads = 512;                  // 16 warps
constexpr int kArWarps = kArThreads / 32;
constexpr int kArMaxHeads = 32;                  // H_q: 2 * H_q split columns <= 64
constexpr int kArNT = 2 * kArMaxHeads / 8;       // n-tiles of 8 split columns
constexpr int kArMaxRows = 128;                  // rows per chunk: 8 m-tiles of 16, two warps each
constexpr int kArMaxMt = kArMaxRows / 16;
constexpr int kArMaxRanks = 16;
constexpr size_t kArSmemBudget = 225 * 1024;

struct ArPlan {
  int nc;      // CTAs of a problem's cluster
  int hpc;     // heads finished per CTA (H_q / nc)
  int e_cap;   // selected rows per chunk, a multiple of 16
  int n_grp;   // kv groups spanned by one CTA's heads (rows of B^V staged: n_grp * d_h)
  int late_bv; // 1: B^V is copied into the spent row buffers after the last chunk (frees its region for rows)
};

// Kv groups spanned by the heads c*hpc .. c*hpc + hpc - 1.
__host__ __device__ inline int ar_groups_of(int G, int hpc, int c) {
  const int h0 = c * hpc, h1 = h0 + hpc - 1;
  return h1 / G - h0 / G + 1;
}

// Shared-memory regions (byte offsets, each 16-byte aligned).
struct ArLayout {
  size_t qb, rows, part, bv, pb, recv, ob, oacc, fl, rows_idx, total;
};
__host__ __device__ inline ArLayout ar_layout(const Shape &s, const ArPlan &pl) {
  const int pk = att_pitch(s.rank_k, 2), pv = att_pitch(s.rank_v, 2), ppb = att_pitch(pl.e_cap, 2);
  const size_t qbytes = (size_t)2 * kArMaxHeads * pk * 2;              // split latent queries
  const size_t rbytes = (size_t)pl.e_cap * (pk + pv) * 2;              // a chunk's C_K and C_V rows
  const size_t part = (size_t)s.n_heads_q * (s.rank_v + 4) * 4;        // this CTA's partials
  const size_t bvb = (size_t)pl.n_grp * s.head_dim * pv * 2;           // rows of B^V
  const size_t obb = (size_t)16 * pv * 2;                               // merged acc, three bf16 terms per head
  const size_t oab = (size_t)16 * pl.n_grp * s.head_dim * 4;           // output products per term
  ArLayout ly;
  size_t o = 0;
  ly.qb = o;
  if (!pl.late_bv) {
    // [qb | ob oacc] [rows | part] [bv] ...
    ly.ob = o;
    ly.oacc = o + obb;
    o += qbytes > obb + oab ? qbytes : obb + oab;
    ly.rows = o;
    o += rbytes > part ? rbytes : part;
    ly.bv = o;
    o += bvb;
  } else {
    // [qb | part] [rows | bv ob oacc] ...: after the last chunk the partials
    // take the query region and B^V, then the output operands, the rows'
    ly.part = o;
    o += qbytes > part ? qbytes : part;
    ly.rows = o;
    ly.bv = o;
    ly.ob = o + bvb;
    ly.oacc = o + bvb + obb;
    o += rbytes > bvb + obb + oab ? rbytes : bvb + obb + oab;
  }
  if (!pl.late_bv) ly.part = ly.rows;
  ly.pb = o;                                                    // [2 * kArMaxHeads][ppb] split weights
  o += (size_t)2 * kArMaxHeads * ppb * 2;
  ly.recv = o;                                                  // [nc][hpc][rv + 4] partials of the heads finished here
  o += part;
  ly.fl = o;
  size_t nf = (size_t)2 * kArMaxMt * kArMaxHeads               // per-m-tile maxima and sums
              + 3 * kArMaxHeads                                 // running max, running sum, rescale
              + (size_t)pl.hpc * (S4R_MAX_SINKS + kArMaxRanks)  // sink logits -> weights; merge weights
              + (size_t)s.n_sink * pl.n_grp * s.head_dim;       // sink values of the output columns
  o += (nf * 4 + 15) / 16 * 16;
  ly.rows_idx = o;                                              // [e_cap] cache row of each staged entry
  o += (size_t)pl.e_cap * 8;
  ly.total = o;
  return ly;
}

// Whether the kernel handles the shape at all (else the per-group kernel of
// k_attend.cuh runs).
__host__ inline bool ar_supported(const Shape &s, int esize) {
  return esize == 2 && s.rank_k % 16 == 0 && s.rank_v % 16 == 0 && s.n_heads_q <= kArMaxHeads &&
         s.n_sink <= S4R_MAX_SINKS && s.head_dim % 8 == 0;
}
// A cluster size suits the kernel when the three split terms of a CTA's
// heads fill one 16-row tile of the output product and they span at most
// two kv groups.
__host__ inline bool ar_plan_ok(const ArPlan &pl) { return pl.hpc >= 1 && 3 * pl.hpc <= 16 && pl.n_grp <= 2; }

// The chunk size is the largest that fits (at most the CTA's rows); B^V is
// prefetched before the wait for the top-k kernel unless copying it after
// the last chunk lets the rows fit in fewer chunks.
__host__ inline ArPlan ar_plan(const Shape &s, int nc) {
  ArPlan pl;
  pl.nc = nc;
  pl.hpc = s.n_heads_q / nc;
  pl.n_grp = 1;
  for (int c = 0; c < nc; ++c) pl.n_grp = smax(pl.n_grp, ar_groups_of(s.group, pl.hpc, c));
  const int64_t per = ceil_div((int64_t)s.top_k + s.local_window, nc);   // rows per CTA at most
  const int want = (int)smin<int64_t>(kArMaxRows, smax<int64_t>(16, (per + 15) / 16 * 16));
  ArPlan best = pl;
  int64_t best_chunks = 0;
  for (int late = 0; late < 2; ++late) {
    ArPlan c = pl;
    c.late_bv = late;
    c.e_cap = want;
    while (c.e_cap > 16 && ar_layout(s, c).total > kArSmemBudget) c.e_cap -= 16;
    const int64_t chunks = ceil_div(per, c.e_cap);
    if (late == 0 || chunks < best_chunks) {
      best = c;
      best_chunks = chunks;
    }
  }
  return best;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}
// Two fp32 values as one 32-bit pair of bf16 (first value in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo_half, float hi_half) {
  const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo_half));
  const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi_half));
  return a | (b << 16);
}
__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__global__ void __launch_bounds__(kArThreads, 1)
attend_rows_kernel(Shape s, ArPlan pl, const int32_t *__restrict__ lengths, const int32_t *__restrict__ idx,
                   const bf16 *__restrict__ coeff_k, const bf16 *__restrict__ coeff_v,
                   const float *__restrict__ qt_all, const bf16 *__restrict__ q, const bf16 *__restrict__ basis_v,
                   const bf16 *__restrict__ sink_k, const bf16 *__restrict__ sink_v, float *__restrict__ out,
                   uint32_t *__restrict__ status) {
  extern __shared__ __align__(16) unsigned char ar_smem[];
  __shared__ __align__(8) uint64_t recv_bar;
  const ArLayout ly = ar_layout(s, pl);
  const int E = pl.e_cap, nc = pl.nc, hpc = pl.hpc;
  const int rk = s.rank_k, rv = s.rank_v, dh = s.head_dim, Dp = s.d_model, ns = s.n_sink, Hq = s.n_heads_q;
  const int G = s.group;
  const int pk = att_pitch(rk, 2), pv = att_pitch(rv, 2), ppb = att_pitch(E, 2), pr = rv + 4;
  bf16 *qb = reinterpret_cast<bf16 *>(ar_smem + ly.qb);
  bf16 *ck = reinterpret_cast<bf16 *>(ar_smem + ly.rows);
  bf16 *cv = ck + (size_t)E * pk;
  float *part = reinterpret_cast<float *>(ar_smem + ly.part);   // after the last chunk: [H_q][pr] = (m, l, -, -, acc)
  bf16 *bvs = reinterpret_cast<bf16 *>(ar_smem + ly.bv);
  bf16 *pb = reinterpret_cast<bf16 *>(ar_smem + ly.pb);
  float *red_m = reinterpret_cast<float *>(ar_smem + ly.fl);    // [kArMaxMt][kArMaxHeads]
  float *red_s = red_m + kArMaxMt * kArMaxHeads;                // [kArMaxMt][kArMaxHeads]
  float *m_run = red_s + kArMaxMt * kArMaxHeads;
  float *l_run = m_run + kArMaxHeads;
  float *resc_s = l_run + kArMaxHeads;                          // rescale of the running sums by the chunk
  float *sw = resc_s + kArMaxHeads;                             // [hpc][S4R_MAX_SINKS]
  float *fw = sw + hpc * S4R_MAX_SINKS;                         // [hpc][kArMaxRanks]
  float *sv = fw + hpc * kArMaxRanks;                           // [ns][n_grp * d_h]
  float *recv = reinterpret_cast<float *>(ar_smem + ly.recv);   // [nc][hpc][pr]
  bf16 *ob = reinterpret_cast<bf16 *>(ar_smem + ly.ob);
  float *oacc = reinterpret_cast<float *>(ar_smem + ly.oacc);
  int64_t *rows_s = reinterpret_cast<int64_t *>(ar_smem + ly.rows_idx);

  const int b = blockIdx.y;
  const uint32_t rank = cluster_ctarank();
  const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  const int h0 = (int)rank * hpc;              // first head finished here
  const int g0 = h0 / G;                       // its kv group
  const int n_grp = (h0 + hpc - 1) / G - g0 + 1;
  const int n_nt = (2 * Hq + 7) / 8;           // n-tiles holding the split columns 2h, 2h + 1

  // The partials of the heads finished here arrive from every rank by bulk
  // copy.  Every rank initialises its barrier before its cluster arrive;
  // ranks copy only after the matching wait.
  if (tid == 0) {
    mbar_init(&recv_bar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&recv_bar, (uint32_t)(nc * hpc * pr * sizeof(float)));
  }
  __syncthreads();
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");

  // 0. Everything that does not depend on the top-k kernel.  The lengths are
  // an input of the call (appends run before it), so the share of the
  // selection list is known here.
  const int64_t L = valid_length(lengths[b], s.cache_rows);
  const int64_t n_top = smin<int64_t>(s.top_k, n_candidates(L, s.local_window));
  const int64_t n_win = smin<int64_t>(s.local_window, L);
  const int64_t n_sel = n_top + n_win;
  const int64_t per = ceil_div(n_sel, nc);
  const int64_t e_begin = smin<int64_t>(n_sel, (int64_t)rank * per);
  const int64_t e_end = smin<int64_t>(n_sel, e_begin + per);
  // Rows of B^V for the heads finished here: warp per row, lane per 16
  // bytes; before the wait, or after the last chunk in the late layout.
  auto copy_bv = [&]() {
    const bf16 *src = basis_v + (int64_t)b * Dp * rv + (int64_t)g0 * dh * rv;
    const int cpr = rv / 8;
    for (int row = wid; row < n_grp * dh; row += kArWarps)
      if (lane < cpr) cp_async16(bvs + (size_t)row * pv + lane * 8, src + (int64_t)row * rv + lane * 8);
    cp_async_commit();
  };
  if (!pl.late_bv) copy_bv();
  {
    // Column n = 2h + term holds head h's latent query as two bf16 terms;
    // columns of heads >= H_q are zero.  float4 j holds k = 4j' .. 4j' + 3
    // of head j / (r_k / 4).
    const int rk4 = rk / 4, nq4 = kArMaxHeads * rk4;
    const float4 *src = reinterpret_cast<const float4 *>(qt_all + (int64_t)b * Hq * rk);
    for (int base = 0; base < nq4; base += 8 * kArThreads) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = base + u * kArThreads + tid;
        v[u] = (j < Hq * rk4) ? __ldcg(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = base + u * kArThreads + tid;
        if (j < nq4) {
          const int h = j / rk4, k = (j - h * rk4) * 4;
          const float hx = bf16_round(v[u].x), hy = bf16_round(v[u].y), hz = bf16_round(v[u].z), hw = bf16_round(v[u].w);
          *reinterpret_cast<uint2 *>(qb + (size_t)(2 * h) * pk + k) = make_uint2(pack_bf16x2(hx, hy), pack_bf16x2(hz, hw));
          *reinterpret_cast<uint2 *>(qb + (size_t)(2 * h + 1) * pk + k) =
              make_uint2(pack_bf16x2(v[u].x - hx, v[u].y - hy), pack_bf16x2(v[u].z - hz, v[u].w - hw));
        }
      }
    }
  }
  {
    // sink logits of the heads finished here (warp per (head, sink)), and the
    // sink values of their output columns
    const float qscale = rsqrtf((float)dh);
    for (int t = wid; t < hpc * ns; t += kArWarps) {
      const int jj = t / ns, tk = t - jj * ns, h = h0 + jj, g = h / G;
      const bf16 *qh = q + (((int64_t)b * s.query_window + s.query_window - 1) * Hq + h) * dh;
      const bf16 *kr = sink_k + ((int64_t)b * ns + tk) * Dp + (int64_t)g * dh;
      float d = 0.f;
      for (int e = lane * 4; e < dh; e += 128) {
        const uint2 qa = *reinterpret_cast<const uint2 *>(qh + e), ka = *reinterpret_cast<const uint2 *>(kr + e);
        const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qa);
        const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&ka);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float2 qf = __bfloat1622float2(q2[u]), kf = __bfloat1622float2(k2[u]);
          d = fmaf(qf.x, kf.x, d);
          d = fmaf(qf.y, kf.y, d);
        }
      }
      d = warp_sum(d);
      if (lane == 0) sw[jj * S4R_MAX_SINKS + tk] = d * qscale;
    }
    const int ncol = n_grp * dh;
    for (int t = tid; t < ns * ncol; t += kArThreads) {
      const int tk = t / ncol, c = t - tk * ncol;
      sv[t] = to_f(sink_v[((int64_t)b * ns + tk) * Dp + (int64_t)g0 * dh + c]);
    }
  }
  if (tid < kArMaxHeads) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.f;
  }
  pdl_wait();      // idx comes from the preceding kernel
  pdl_trigger();

  const int32_t *idx_b = idx + (int64_t)b * s.top_k;
  const bf16 *ckb = coeff_k + (int64_t)b * s.cache_rows * rk;
  const bf16 *cvb = coeff_v + (int64_t)b * s.cache_rows * rv;

  // acc^T tile: warp w owns latent-column tile w (r_v / 16 <= 16) for every
  // n-tile; lane (gq, tq) holds latent columns gq, gq + 8 and split columns
  // 2tq, 2tq + 1 of each, the two terms of head 4 * nt + tq.
  float acc[kArNT][4];
#pragma unroll
  for (int c = 0; c < kArNT; ++c)
#pragma unroll
    for (int d = 0; d < 4; ++d) acc[c][d] = 0.f;
  const int lm = lane >> 3, lr = lane & 7;   // ldmatrix: matrix of this lane's row address, row within it
  const int mt = wid >> 1, nh = wid & 1;     // logits: m-tile (16 rows) and half of the n-tiles of this warp

  for (int64_t c0 = e_begin; c0 < e_end; c0 += E) {
    const int n_e = (int)smin<int64_t>(E, e_end - c0);
    const int n_e16 = (n_e + 15) & ~15;
    __syncthreads();   // the previous chunk's rows, weights and maxima are consumed
    // Warp w takes rows w, w + 16, ...: every lane reads the same idx entry
    // (one broadcast load each), lane 0 records the row for the logits, and
    // the lanes copy the C_K rows, then the C_V rows, 16 bytes each; rows not
    // selected and the padding up to 16 rows are zeroed, so products over
    // them are 0.
    int64_t rr[kArMaxRows / kArWarps];
#pragma unroll
    for (int u = 0; u < kArMaxRows / kArWarps; ++u) {
      const int e = wid + u * kArWarps;
      int64_t row = -1;
      if (e < n_e) {
        row = att_entry_row(idx_b, n_top, L, n_win, c0 + e, s.n_sink);
        if (row < 0 || row >= L) row = -1;   // never produced by the top-k kernel
      }
      rr[u] = row;
      if (lane == 0 && e < n_e16) rows_s[e] = row;
    }
#pragma unroll
    for (int u = 0; u < kArMaxRows / kArWarps; ++u) {
      const int e = wid + u * kArWarps;
      if (e < n_e16 && lane < rk / 8) {
        bf16 *dst = ck + (size_t)e * pk + lane * 8;
        if (rr[u] >= 0) cp_async16(dst, ckb + rr[u] * rk + lane * 8);
        else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
#pragma unroll
    for (int u = 0; u < kArMaxRows / kArWarps; ++u) {
      const int e = wid + u * kArWarps;
      if (e < n_e16 && lane < rv / 8) {
        bf16 *dst = cv + (size_t)e * pv + lane * 8;
        if (rr[u] >= 0) cp_async16(dst, cvb + rr[u] * rv + lane * 8);
        else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
    cp_async_wait_group<1>();   // this thread's C_K (and B^V) copies have landed
    __syncthreads();            // and everyone's

    // Logits of rows 16mt .. 16mt + 15 and n-tiles 4nh .. 4nh + 3.
    const bool have_mt = mt * 16 < n_e16;
    float lg[kArNT / 2][2];
    {
      float c[kArNT / 2][4];
#pragma unroll
      for (int j = 0; j < kArNT / 2; ++j)
#pragma unroll
        for (int d = 0; d < 4; ++d) c[j][d] = 0.f;
      if (have_mt && 4 * nh < n_nt) {
        const bf16 *a_row = ck + (size_t)(mt * 16 + (lm & 1) * 8 + lr) * pk + (lm >> 1) * 8;
        const bf16 *b_row = qb + (size_t)(nh * 32 + (lm >> 1) * 8 + lr) * pk + (lm & 1) * 8;
#pragma unroll 2
        for (int ks = 0; ks < rk / 16; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(a_row + ks * 16, a0, a1, a2, a3);
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
            if (4 * nh + 2 * pp < n_nt) {
              uint32_t b0, b1, b2, b3;
              ldsm_x4(b_row + (size_t)(pp * 16) * pk + ks * 16, b0, b1, b2, b3);
              mma_bf16_16816(c[2 * pp], a0, a1, a2, a3, b0, b1);
              mma_bf16_16816(c[2 * pp + 1], a0, a1, a2, a3, b2, b3);
            }
          }
        }
      }
      const int e0 = mt * 16 + gq, e1 = e0 + 8;
      const bool ok0 = have_mt && e0 < n_e && rows_s[e0] >= 0;
      const bool ok1 = have_mt && e1 < n_e && rows_s[e1] >= 0;
#pragma unroll
      for (int j = 0; j < kArNT / 2; ++j) {
        lg[j][0] = ok0 ? c[j][0] + c[j][1] : -INFINITY;
        lg[j][1] = ok1 ? c[j][2] + c[j][3] : -INFINITY;
      }
    }
    // Maximum of each head over the m-tile's 16 rows (the 8 lanes sharing tq).
    if (mt < kArMaxMt) {
#pragma unroll
      for (int j = 0; j < kArNT / 2; ++j) {
        float v = fmaxf(lg[j][0], lg[j][1]);
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        if (gq == 0) red_m[mt * kArMaxHeads + (nh * 4 + j) * 4 + tq] = v;
      }
    }
    __syncthreads();
    // Running max per head after the chunk, and the rescale of what came before.
    if (tid < kArMaxHeads) {
      const int h = tid;
      const float m_old = m_run[h];
      float m = m_old;
#pragma unroll
      for (int t = 0; t < kArMaxMt; ++t) m = fmaxf(m, red_m[t * kArMaxHeads + h]);
      resc_s[h] = (m_old == -INFINITY) ? 0.f : __expf(m_old - m);
      m_run[h] = m;
    }
    __syncthreads();
    // Weights and their sums.  The weight of row j of m-tile t goes to entry
    // 16t + 2j (rows j < 8) or 16t + 2(j - 8) + 1 of the value product's K
    // order, so each lane stores its two rows as one 32-bit pair.
    if (mt < kArMaxMt) {
#pragma unroll
      for (int j = 0; j < kArNT / 2; ++j) {
        const int h = (nh * 4 + j) * 4 + tq;
        const float m = m_run[h];
        const float p0 = (m == -INFINITY) ? 0.f : __expf(lg[j][0] - m);
        const float p1 = (m == -INFINITY) ? 0.f : __expf(lg[j][1] - m);
        if (have_mt) {
          const float h0f = bf16_round(p0), h1f = bf16_round(p1);
          *reinterpret_cast<uint32_t *>(pb + (size_t)(2 * h) * ppb + mt * 16 + 2 * gq) = pack_bf16x2(h0f, h1f);
          *reinterpret_cast<uint32_t *>(pb + (size_t)(2 * h + 1) * ppb + mt * 16 + 2 * gq) =
              pack_bf16x2(p0 - h0f, p1 - h1f);
        }
        float sm = p0 + p1;
        sm += __shfl_xor_sync(0xffffffffu, sm, 4);
        sm += __shfl_xor_sync(0xffffffffu, sm, 8);
        sm += __shfl_xor_sync(0xffffffffu, sm, 16);
        if (gq == 0) red_s[mt * kArMaxHeads + h] = sm;
      }
    }
    cp_async_wait_group<0>();   // this thread's C_V copies have landed
    __syncthreads();            // and everyone's; the weights and sums are written
    if (tid < kArMaxHeads) {
      float sum = 0.f;
#pragma unroll
      for (int t = 0; t < kArMaxMt; ++t) sum += red_s[t * kArMaxHeads + tid];
      l_run[tid] = l_run[tid] * resc_s[tid] + sum;
    }
    // acc^T += C_V^T . W over the chunk's rows, in the permuted K order: K
    // entry 2j of step ks is row 16ks + j, entry 2j + 1 is row 16ks + j + 8.
    if (wid < rv / 16) {
      const int kap = ((lm & 2) ? 8 : 0) + lr;                   // K entry of this lane's A row address
      const int e_of_kap = (kap & 1) ? (kap >> 1) + 8 : (kap >> 1);
#pragma unroll
      for (int c = 0; c < kArNT; ++c) {
        const float sc = resc_s[c * 4 + tq];
#pragma unroll
        for (int d = 0; d < 4; ++d) acc[c][d] *= sc;
      }
      const bf16 *a_row = cv + (size_t)e_of_kap * pv + wid * 16 + (lm & 1) * 8;
      const bf16 *b_row = pb + (size_t)((lm >> 1) * 8 + lr) * ppb + (lm & 1) * 8;
      for (int ks = 0; ks < n_e16 / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(a_row + (size_t)(ks * 16) * pv, a0, a1, a2, a3);
#pragma unroll
        for (int pp = 0; pp < kArNT / 2; ++pp) {
          if (2 * pp < n_nt) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(b_row + (size_t)(pp * 16) * ppb + ks * 16, b0, b1, b2, b3);
            mma_bf16_16816(acc[2 * pp], a0, a1, a2, a3, b0, b1);
            mma_bf16_16816(acc[2 * pp + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
    }
  }
  __syncthreads();   // every warp is done with the row buffers, which now take the partials
  if (wid < rv / 16) {
#pragma unroll
    for (int c = 0; c < kArNT; ++c) {
      const int h = c * 4 + tq;
      if (h < Hq) {
        part[(size_t)h * pr + 4 + wid * 16 + gq] = acc[c][0] + acc[c][1];
        part[(size_t)h * pr + 4 + wid * 16 + gq + 8] = acc[c][2] + acc[c][3];
      }
    }
  }
  if (tid < Hq) {
    part[(size_t)tid * pr] = m_run[tid];
    part[(size_t)tid * pr + 1] = l_run[tid];
  }
  if (pl.late_bv) copy_bv();   // the row buffers are spent; lands while the partials are exchanged
  // 2. Push the partial rows of the heads rank r finishes into rank r's
  // receive buffer (slot of this rank); the bulk copies read what the
  // threads just wrote.
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");   // every rank's barrier is initialised
  if (tid < nc)
    bulk_copy_to_peer(cluster_map(recv + (size_t)rank * hpc * pr, (uint32_t)tid), part + (size_t)tid * hpc * pr,
                      (uint32_t)(hpc * pr * sizeof(float)), cluster_map(&recv_bar, (uint32_t)tid));
  const bool got = mbar_wait(&recv_bar, 0, status);   // every rank's partials of the heads finished here
  // Every copy into this CTA is done.  A sender learns that its own copies
  // have been read only from the receivers, so no CTA leaves before all have
  // arrived (the wait is the kernel's last step).  The arrive publishes no
  // data, hence relaxed.
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // Merge weights of the heads finished here (warp per head, ranks = lanes).
  for (int jj = wid; jj < hpc; jj += kArWarps) {
    float mr = -INFINITY, lr_ = 0.f;
    if (lane < nc && got) {
      mr = recv[((size_t)lane * hpc + jj) * pr];
      lr_ = recv[((size_t)lane * hpc + jj) * pr + 1];
    }
    float M = mr;
    for (int tk = lane; tk < ns; tk += 32) M = fmaxf(M, sw[jj * S4R_MAX_SINKS + tk]);
    M = warp_max(M);
    const float fr = (mr == -INFINITY) ? 0.f : __expf(mr - M);
    float den = lr_ * fr;
    for (int tk = lane; tk < ns; tk += 32) den += __expf(sw[jj * S4R_MAX_SINKS + tk] - M);
    den = warp_sum(den);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    if (lane < nc) fw[jj * kArMaxRanks + lane] = fr * inv;
    __syncwarp();
    for (int tk = lane; tk < ns; tk += 32)
      sw[jj * S4R_MAX_SINKS + tk] = __expf(sw[jj * S4R_MAX_SINKS + tk] - M) * inv;
  }
  __syncthreads();
  // acc_h = sum_r f_r acc_{r,h}, written as three bf16 terms (rows 3jj + term
  // of the output product's A operand; the other rows are zero).
  {
    const int rv4 = rv / 4;
    for (int t = tid; t < 16 * rv4; t += kArThreads) {
      const int row = t / rv4, k4 = t - row * rv4, jj = row / 3, term = row - 3 * jj;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (jj < hpc) {
        for (int r = 0; r < nc; ++r) {
          const float f = fw[jj * kArMaxRanks + r];
          const float4 v = *reinterpret_cast<const float4 *>(recv + ((size_t)r * hpc + jj) * pr + 4 + 4 * k4);
          o.x = fmaf(f, v.x, o.x);
          o.y = fmaf(f, v.y, o.y);
          o.z = fmaf(f, v.z, o.z);
          o.w = fmaf(f, v.w, o.w);
        }
        // term 0: bf16(x); term 1: bf16(x - t0); term 2: bf16(x - t0 - t1)
        float x[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float rest = x[u];
          for (int q = 0; q < term; ++q) rest -= bf16_round(rest);
          x[u] = rest;
        }
        o = make_float4(x[0], x[1], x[2], x[3]);
      }
      *reinterpret_cast<uint2 *>(ob + (size_t)row * pv + 4 * k4) = make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w));
    }
  }
  cp_async_wait_group<0>();   // B^V (when no chunk ran)
  __syncthreads();
  // Output product oacc[row][col] = A[row] . B^V[g0*dh + col] over r_v
  // (mma.sync; warp per 8 output columns), then
  // out[h][e] = sum_term oacc[3jj + term][gi*dh + e] + sum_t w_t sink_v[t][g*dh + e].
  {
    const int ncol = n_grp * dh;
    for (int nt = wid; nt < ncol / 8; nt += kArWarps) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      const bf16 *a_row = ob + (size_t)((lm & 1) * 8 + lr) * pv + (lm >> 1) * 8;
      const bf16 *b_row = bvs + (size_t)(nt * 8 + lr) * pv + (lm & 1) * 8;
      for (int ks = 0; ks < rv / 16; ++ks) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        ldsm_x4(a_row + ks * 16, a0, a1, a2, a3);
        ldsm_x4(b_row + ks * 16, b0, b1, b2, b3);   // matrices 2, 3 repeat 0, 1
        mma_bf16_16816(c, a0, a1, a2, a3, b0, b1);
      }
      oacc[(size_t)gq * ncol + nt * 8 + 2 * tq] = c[0];
      oacc[(size_t)gq * ncol + nt * 8 + 2 * tq + 1] = c[1];
      oacc[(size_t)(gq + 8) * ncol + nt * 8 + 2 * tq] = c[2];
      oacc[(size_t)(gq + 8) * ncol + nt * 8 + 2 * tq + 1] = c[3];
    }
    __syncthreads();
    for (int item = tid; item < hpc * dh; item += kArThreads) {
      const int jj = item / dh, e = item - jj * dh, col = ((h0 + jj) / G - g0) * dh + e;
      float o = (oacc[(size_t)(3 * jj) * ncol + col] + oacc[(size_t)(3 * jj + 1) * ncol + col]) +
                oacc[(size_t)(3 * jj + 2) * ncol + col];
      for (int tk = 0; tk < ns; ++tk) o = fmaf(sw[jj * S4R_MAX_SINKS + tk], sv[(size_t)tk * ncol + col], o);
      out[((int64_t)b * Hq + h0 + jj) * dh + e] = o;
    }
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace s4r
