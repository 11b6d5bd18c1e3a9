// k_project.cuh -- query projection into the key basis.
//
// "Core claim" of the S4R review page: at decoding, queries are projected into
// the key subspace; the sliding query window is then scored in latent space
// (Eqs. 8-10).  Every per-head projection
//     p[w][h][c] = q[w][h] . B^K[g*d_h : (g+1)*d_h][c],   g = h / G,
// is computed once, and from it
//   * CONCAT rows:   C_Q[w*G + j] = sum_g p[w][g*G + j]   (row = Q'[w][j] . B^K)
//   * PER_HEAD rows: C_Q[w*H_q + h] = p[w][h]
//   * qt[h] = p[W-1][h] / sqrt(d_h), the current query in latent form for the
//     absorbed exact-attention logits q . (c B^T) = (q B) . c.
// Grid: (cluster rank, 64-column block, 16-row block x problem).  The CTAs of
// a cluster cover the kv groups (rank, rank + cluster size, ...).  Products of
// two storage values are exact in fp32; each dot product sums 64-term fp32
// chunks in fp64.  CONCAT rows are summed over the groups by rank 0, which
// reads the other ranks' fp64 partials through distributed shared memory.
// The CTA that finishes a row writes
//   * cq  [R][r_k] fp32 (natural-log units), read by the CUDA-core scoring;
//   * cqs  the shared-memory image of the tensor-core operand: C_Q * log2(e)
//     split into three bf16 terms hi + mid + lo (rows term*R + i), K-major,
//     128-byte swizzled, one 3R x 64 block per 64 columns.
#pragma once
#include "common.cuh"
#include "k_score_tc.cuh"
#include "umma.cuh"

namespace s4r {

constexpr int kProjThreads = 128;
constexpr int kProjColBlock = 64;   // columns per CTA (= one 128-byte swizzle row of bf16)
constexpr int kProjRowBlock = 16;   // per-head rows (w, j) per CTA
constexpr int kProjMaxCluster = 8;

// Shared-memory image of the split C_Q operand: bytes per 64-column block.
__host__ __device__ constexpr int cqs_block_bytes(int R) { return 3 * R * 128; }
__host__ __device__ inline int proj_cluster(int n_heads_kv) { return n_heads_kv < kProjMaxCluster ? n_heads_kv : kProjMaxCluster; }

// Write scoring row i, columns c0 .. c0+63, from its fp64 values x (already
// scaled by 1/sqrt(r)): fp32 copy for the CUDA-core path and the bf16 split.
__device__ __forceinline__ void proj_finish(double x, int b, int R, int r, int i, int c, int kk, float *cq,
                                            unsigned char *blk, int64_t copy_stride) {
  if (c < r) cq[((int64_t)b * R + i) * r + c] = (float)x;
  // y = x log2(e) as y1 + y2 (fp32 pair, |y2| <= ulp(y1)/2), then three bf16
  // terms whose residuals are exact fp32 differences.
  const double y = x * 1.4426950408889634;
  const float y1 = (float)y;
  const float y2 = (float)(y - (double)y1);
  const bf16 hi = __float2bfloat16_rn(y1);
  const float r1 = (y1 - __bfloat162float(hi)) + y2;
  const bf16 mid = __float2bfloat16_rn(r1);
  const bf16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
#pragma unroll
  for (int cp = 0; cp < kCqsCopies; ++cp) {
    unsigned char *dst = blk + cp * copy_stride;
    *reinterpret_cast<bf16 *>(dst + sw128_offset(i, kk)) = hi;
    *reinterpret_cast<bf16 *>(dst + sw128_offset(R + i, kk)) = mid;
    *reinterpret_cast<bf16 *>(dst + sw128_offset(2 * R + i, kk)) = lo;
  }
}

// Per-head results of group g: qt (current query, scaled by 1/sqrt(d_h)) and,
// for PER_HEAD rows, the finished scoring rows.
__device__ __forceinline__ void proj_head_writes(const Shape &s, const double (&acc)[2][4], int g, int b, int pr0,
                                                 int c0, double scale, float *cq, unsigned char *blk, float *qt) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int G = s.group, W = s.query_window, Hq = s.n_heads_q, dh = s.head_dim, r = s.rank_k, R = s.n_rows;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int row = pr0 + ty + 8 * i;
    if (row >= W * G) continue;
    const int w = row / G, j = row - w * G, h = g * G + j;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int kk = tx + 16 * jj, c = c0 + kk;
      const double v = acc[i][jj];
      if (w == W - 1 && c < r) qt[((int64_t)b * Hq + h) * r + c] = (float)(v / sqrt((double)dh));
      if (s.row_mode == S4R_ROWS_PER_HEAD) proj_finish(c < r ? v * scale : 0.0, b, R, r, w * Hq + h, c, kk, cq, blk, (int64_t)s.batch * stc_b_bytes(R, r));
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kProjThreads)
project_kernel(Shape s, const T *__restrict__ q, const T *__restrict__ basis_k, float *__restrict__ cq,
               unsigned char *__restrict__ cqs, float *__restrict__ qt, double *__restrict__ row_sum,
               uint32_t *__restrict__ ehist, unsigned int *__restrict__ counters) {
  // Raw storage-type slices, copied with 16-byte cp.async (all in flight at once).
  __shared__ __align__(16) T qraw[kProjRowBlock][128];                  // per-head query rows, 128 of d_h
  __shared__ __align__(16) T braw[128][kProjColBlock + 16 / sizeof(T)];  // basis slice (padded rows)
  constexpr int V = Vec16<T>::n;
  const int rank = (int)blockIdx.x, n_rank = (int)gridDim.x, cb = blockIdx.y;
  // Programmatic launch: this kernel may start while the previous decode
  // call's attention kernel still runs, but only once every CTA of it has
  // passed its own wait and trigger.  Both attention kernels read qt only
  // before that point, and every other buffer written here was last read by
  // kernels that completed before the attention kernel passed its wait; so
  // this kernel writes without waiting.  It still waits at its end: its
  // completion then implies the attention kernel's, so the next kernels of
  // this call (the top-k writes idx, which that attention kernel reads) are
  // ordered after it.  The next kernel (scoring) only reads caller inputs
  // before its own wait, so it may be released right away.
  const bool early = (s.n_heads_kv - rank + n_rank - 1) / n_rank <= 1;
  pdl_trigger();
  const int n_rb = (int)ceil_div((int64_t)s.query_window * s.group, kProjRowBlock);
  const int rb = blockIdx.z % n_rb, b = blockIdx.z / n_rb;
  const int G = s.group, W = s.query_window, Hq = s.n_heads_q, dh = s.head_dim, r = s.rank_k;
  const int R = s.n_rows;
  const int c0 = cb * kProjColBlock;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 8: 2 rows x 4 cols each
  const T *qb = q + (int64_t)b * W * Hq * dh;
  const T *Bb = basis_k + (int64_t)b * s.d_model * r;
  const double scale = 1.0 / sqrt((double)r);
  unsigned char *blk = cqs + ((int64_t)b * gridDim.y + cb) * cqs_block_bytes(R);
  // Reset the per-call accumulators of the tensor-core scoring kernel.
  if (rank == 0 && cb == 0 && rb == 0) {
    for (int e = threadIdx.x; e < kStcSumSlots * R; e += blockDim.x) row_sum[(int64_t)b * kStcSumSlots * R + e] = 0.0;
    for (int e = threadIdx.x; e < kExpBins; e += blockDim.x) ehist[(int64_t)b * kExpBins + e] = 0u;
    if (threadIdx.x == 0) counters[b] = 0u;
  }
  const int n_prow = W * G;  // per-head rows (w, j) of one group
  const int pr0 = rb * kProjRowBlock;
  double gsum[2][4];          // sum over this CTA's groups (CONCAT rows)
  double keep[2][4] = {};     // the single group's results (early CTAs)
  int g_keep = rank;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) gsum[i][j] = 0.0;
  for (int g = rank; g < s.n_heads_kv; g += n_rank) {
    double acc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int t0 = 0; t0 < dh; t0 += 128) {
      const int tn = smin(128, dh - t0);  // a multiple of 8
      __syncthreads();
      for (int e = threadIdx.x; e < kProjRowBlock * (128 / V); e += blockDim.x) {
        const int pr = e / (128 / V), cc = e - pr * (128 / V);
        const int row = pr0 + pr;
        T *dst = &qraw[pr][cc * V];
        if (row < n_prow && cc * V < tn) {
          const int w = row / G, j = row - w * G;
          cp_async16(dst, qb + ((int64_t)w * Hq + g * G + j) * dh + t0 + cc * V);
        } else {
          *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      for (int e = threadIdx.x; e < 128 * (kProjColBlock / V); e += blockDim.x) {
        const int t = e / (kProjColBlock / V), cc = e - t * (kProjColBlock / V);
        T *dst = &braw[t][cc * V];
        if (t < tn && c0 + cc * V < r)   // r % 8 == 0, so a chunk never straddles r
          cp_async16(dst, Bb + (int64_t)(g * dh + t0 + t) * r + c0 + cc * V);
        else
          *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
      cp_async_wait_all();
      __syncthreads();
#pragma unroll
      for (int h0 = 0; h0 < 128; h0 += 64) {
        float pp[2][4] = {};
#pragma unroll 16
        for (int k = h0; k < h0 + 64; ++k) {
          float a[2], bb[4];
#pragma unroll
          for (int i = 0; i < 2; ++i) a[i] = to_f(qraw[ty + 8 * i][k]);
#pragma unroll
          for (int j = 0; j < 4; ++j) bb[j] = to_f(braw[k][tx + 16 * j]);
#pragma unroll
          for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) pp[i][j] = fmaf(a[i], bb[j], pp[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] += (double)pp[i][j];
      }
    }
    if (early) {
      // Single group: keep its results; the writes wait below.
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          keep[i][jj] = acc[i][jj];
          gsum[i][jj] += acc[i][jj];
        }
      g_keep = g;
    } else {
      proj_head_writes(s, acc, g, b, pr0, c0, scale, cq, blk, qt);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) gsum[i][jj] += acc[i][jj];
    }
  }
  // CONCAT: rank 0 sums the ranks' group sums (fixed rank order).  The
  // exchange needs nothing from the previous call, so it runs before the
  // wait; only the stores follow it.  The group sums reuse the basis staging
  // buffer, which is no longer read.
  double x[2][4] = {};
  if (s.row_mode == S4R_ROWS_CONCAT) {
    static_assert(sizeof(double) * kProjRowBlock * kProjColBlock <= sizeof(T) * 128 * (kProjColBlock + 16 / sizeof(T)),
                  "group sums must fit the staging buffer");
    double(*part)[kProjColBlock] = reinterpret_cast<double(*)[kProjColBlock]>(&braw[0][0]);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) part[ty + 8 * i][tx + 16 * jj] = gsum[i][jj];
    cluster_sync();
    if (rank == 0) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int kk = tx + 16 * jj;
          for (int rr = 0; rr < n_rank; ++rr) {
            const uint32_t a = cluster_map(&part[ty + 8 * i][kk], (uint32_t)rr);
            double v;
            asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(a) : "memory");
            x[i][jj] += v;
          }
        }
    }
    cluster_sync();  // rank 0 has read every partial
  }
  if (early) proj_head_writes(s, keep, g_keep, b, pr0, c0, scale, cq, blk, qt);
  if (s.row_mode == S4R_ROWS_CONCAT && rank == 0)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int row = pr0 + ty + 8 * i;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int kk = tx + 16 * jj, c = c0 + kk;
        if (row < W * G) proj_finish(c < r ? x[i][jj] * scale : 0.0, b, R, r, row, c, kk, cq, blk, (int64_t)s.batch * stc_b_bytes(R, r));
      }
    }
  pdl_wait();   // complete only after the previous call's attention kernel (see above)
}

}  // namespace s4r
