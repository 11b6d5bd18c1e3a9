// k_basis.cuh -- prefill bases on the GPU: sample, normalise, truncated SVD.
//
// S4R review page, "What carries the argument" and the Referee Report's
// summary (Eqs. 1-2): the key (or value) basis of a problem is the set of
// top-r right singular vectors of a sampled, token-wise normalised set of
// non-sink states; "Core claim" and the free-parameter list fix the sample:
// T' non-sink tokens split 7:3 between the most recent rows and rows spaced
// evenly over the older ones.
//
// Readings the page leaves open (the fp64 oracle takes the same ones):
//   * the sample has n = min(T', L - s) rows; the recent share is the last
//     (7n + 5) div 10 rows (0.7 n rounded half up), the other n_u rows are
//     s + floor(j * span / n_u), j < n_u, span = L - s - recent share;
//   * each sampled row is scaled to unit Euclidean norm (zero rows stay 0);
//   * columns are ordered by decreasing singular value and signed so that
//     the entry of largest magnitude (lowest index on ties) is positive.
//
// All arithmetic is fp64.  The SVD goes through the smaller Gram matrix of
// the sample, m = min(T', D') rounded up to even: A A^T (T' x T', then
// B = A^T U Sigma^-1) when T' <= D', else A^T A (D' x D', B = its
// eigenvectors).  Its eigenvectors come from a two-sided cyclic Jacobi
// method in parallel rounds: the m/2 disjoint pairs of a round (round-robin
// order, every pair once per sweep) rotate together, so M' = J^T M J splits
// into independent 2x2 blocks R_a^T M[a][b] R_b.  The matrix is stored in
// the round's slot order (pair a in slots 2a, 2a+1), so a block is two
// 16-byte loads; each round writes its result into the other buffer already
// in the next round's slot order, and keeps only the upper blocks' work
// (the lower ones are their transposes).  The eigenvectors are kept as the
// rows of V^T in the same slot order, so their rotation is a pair of
// contiguous rows.  The rounds of all problems are separated by a grid-wide
// barrier of one cooperative launch.  The sweep in which every pair meets
// an off-diagonal entry below 1e-8 of its diagonal scale is the last one:
// its rotations leave them near their squares.
// Near the rank cut the eigenvalues of the workloads' samples differ by
// 1e-5 .. 1e-3 of the largest, so single precision would mix kept and
// dropped directions; fp64 keeps them apart to ~1e-10.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace s4r {

constexpr int kBasisMaxSweeps = 30;
constexpr double kJacobiTol = 1e-12;   // rotate while |a_pq| > tol * sqrt(a_pp a_qq)
// A sweep in which no pair starts above this relative size leaves every
// off-diagonal entry near its square (quadratic convergence): the last sweep.
constexpr double kJacobiLastSweep = 1e-8;

struct BasisShape {
  int32_t P;         // problems
  int32_t D;         // D'
  int32_t r;         // rank
  int32_t s;         // sinks
  int32_t T;         // requested sample rows T'
  int32_t m;         // Gram dimension (even)
  int32_t t_side;    // 1: Gram of the rows (A A^T), 0: Gram of the columns (A^T A)
  int64_t state_rows;
};

// Control words at the head of the workspace.  word 0 is the sticky status.
struct BasisCtl {
  uint32_t status;
  uint32_t bar;                   // grid barrier arrivals (monotone)
  uint32_t final_buf;             // buffer of M and V^T holding the converged result
  uint32_t pad;
  uint32_t rot[kBasisMaxSweeps];  // CTAs that met a pair above kJacobiLastSweep in sweep i
};

// Row of sample j (< n) of a problem with L rows ("Core claim", 7:3 split).
__host__ __device__ __forceinline__ int64_t basis_sample_row(int64_t L, int64_t s, int64_t n, int64_t j) {
  const int64_t n_recent = (7 * n + 5) / 10;
  const int64_t n_uniform = n - n_recent;
  if (j < n_uniform) {
    const int64_t span = (L - s) - n_recent;
    return s + (j * span) / n_uniform;
  }
  return L - n_recent + (j - n_uniform);
}

// Round-robin schedule (circle method): player m-1 is fixed, the others sit
// on a circle of n1 = m-1 places; in round k (< n1) pair 0 is (m-1, k) and
// pair a >= 1 is ((k+a) mod n1, (k-a) mod n1).  Every pair meets once in n1
// rounds.  Pair a occupies slots 2a (first) and 2a+1 (second).
__host__ __device__ __forceinline__ int jac_player(int m, int k, int u) {
  const int n1 = m - 1, a = u >> 1;
  if ((u & 1) == 0) return a == 0 ? m - 1 : (k + a) % n1;
  return a == 0 ? k % n1 : (k - a + n1) % n1;
}
__host__ __device__ __forceinline__ int jac_slot(int m, int k, int x) {
  const int n1 = m - 1, h = m / 2;
  if (x == m - 1) return 0;
  const int d = ((x - k) % n1 + n1) % n1;
  if (d == 0) return 1;
  if (d <= h - 1) return 2 * d;
  return 2 * (n1 - d) + 1;
}

__device__ __forceinline__ int64_t basis_n(const BasisShape &bs, const int32_t *lengths, int p) {
  const int64_t L = lengths[p];
  if (L < 0 || L > bs.state_rows) return 0;
  const int64_t avail = L - bs.s;
  return avail < 0 ? 0 : (avail < bs.T ? avail : (int64_t)bs.T);
}

// 1. Sampled rows and their inverse norms (one warp per sample row); zeroes
// the control words.
template <typename T>
__global__ void __launch_bounds__(256) basis_prep_kernel(BasisShape bs, const int32_t *__restrict__ lengths,
                                                         const T *__restrict__ states, int64_t *__restrict__ rows,
                                                         double *__restrict__ inv, BasisCtl *ctl) {
  const int p = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (p == 0 && blockIdx.x == 0) {
    for (int i = threadIdx.x; i < kBasisMaxSweeps; i += blockDim.x) ctl->rot[i] = 0u;
    if (threadIdx.x == 0) {
      ctl->bar = 0u;
      ctl->final_buf = 0u;
    }
  }
  const int64_t Lraw = lengths[p];
  const int64_t n = basis_n(bs, lengths, p);
  if (blockIdx.x == 0 && threadIdx.x == 0 && (Lraw < 0 || Lraw > bs.state_rows || n < bs.r))
    set_status(&ctl->status, kDevStatusCheck);
  const int64_t j = (int64_t)blockIdx.x * 8 + warp;
  if (j >= bs.T) return;
  int64_t row = -1;
  double ss = 0.0;
  if (j < n) {
    row = basis_sample_row(Lraw, bs.s, n, j);
    const T *x = states + ((int64_t)p * bs.state_rows + row) * bs.D;
    for (int d = lane; d < bs.D; d += 32) {
      const double v = (double)to_f(x[d]);
      ss = fma(v, v, ss);
    }
    ss = warp_sum(ss);
  }
  if (lane == 0) {
    rows[(int64_t)p * bs.T + j] = row;
    inv[(int64_t)p * bs.T + j] = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;
  }
}

// Normalised sample entry a[j][d] (0 outside the sample).
template <typename T>
__device__ __forceinline__ double basis_a(const BasisShape &bs, const T *states, const int64_t *rows_p,
                                          const double *inv_p, int p, int64_t j, int d) {
  if (j >= bs.T || d >= bs.D) return 0.0;
  const int64_t row = rows_p[j];
  if (row < 0) return 0.0;
  return (double)to_f(states[((int64_t)p * bs.state_rows + row) * bs.D + d]) * inv_p[j];
}

// 2. Gram matrix M (buffer 0, slot order of round 0) and V^T = I.  32 x 32 output tile per CTA, four
// outputs per thread, inner dimension in chunks of 32 staged in shared
// memory.  Gram of the rows: M[i][j] = sum_d a[i][d] a[j][d]; of the
// columns: M[i][j] = sum_t a[t][i] a[t][j].
template <typename T>
__global__ void __launch_bounds__(256) basis_gram_kernel(BasisShape bs, const T *__restrict__ states,
                                                         const int64_t *__restrict__ rows,
                                                         const double *__restrict__ inv, double *__restrict__ M,
                                                         double *__restrict__ V) {
  __shared__ double a_s[32][33], b_s[32][33];
  const int p = blockIdx.z;
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // ty < 8
  const int m = bs.m;
  const int64_t *rows_p = rows + (int64_t)p * bs.T;
  const double *inv_p = inv + (int64_t)p * bs.T;
  const int K = bs.t_side ? bs.D : bs.T;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int e = threadIdx.x; e < 32 * 32; e += blockDim.x) {
      if (bs.t_side) {
        const int ii = e >> 5, kk = e & 31;   // consecutive threads walk d
        a_s[ii][kk] = basis_a(bs, states, rows_p, inv_p, p, i0 + ii, k0 + kk);
        b_s[ii][kk] = basis_a(bs, states, rows_p, inv_p, p, j0 + ii, k0 + kk);
      } else {
        const int kk = e >> 5, ii = e & 31;   // consecutive threads walk d
        a_s[ii][kk] = basis_a(bs, states, rows_p, inv_p, p, k0 + kk, i0 + ii);
        b_s[ii][kk] = basis_a(bs, states, rows_p, inv_p, p, k0 + kk, j0 + ii);
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const double bv = b_s[tx][kk];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = fma(a_s[ty + 8 * u][kk], bv, acc[u]);
    }
    __syncthreads();
  }
  // Round 0's slot order; row slot(i) of V^T starts as e_i.
  double *Mp = M + (int64_t)p * 2 * m * m;
  double *Vp = V + (int64_t)p * 2 * m * m;
  const int sj = (j0 + tx < m) ? jac_slot(m, 0, j0 + tx) : 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty + 8 * u, j = j0 + tx;
    if (i < m && j < m) {
      const int si = jac_slot(m, 0, i);
      Mp[(int64_t)si * m + sj] = acc[u];
      Vp[(int64_t)si * m + j] = (i == j) ? 1.0 : 0.0;
    }
  }
}

// Grid-wide barrier number `gen` (1, 2, ...) of a cooperative launch on a
// monotone arrival counter; bounded wait, false on timeout.
__device__ __forceinline__ bool basis_grid_sync(BasisCtl *ctl, uint32_t gen, int *flag_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    atomicAdd(&ctl->bar, 1u);
    const uint32_t target = gen * gridDim.x;
    const long long limit = wait_limit();
    const long long t0 = clock64();
    while (true) {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&ctl->bar) : "memory");
      if (v >= target) break;
      if (clock64() - t0 > limit) {
        set_status(&ctl->status, kDevStatusTimeout);
        ok = 0;
        break;
      }
      __nanosleep(64);   // fewer polls on the counter line while the arrivals land
    }
    *flag_smem = ok;
  }
  __syncthreads();
  return *flag_smem != 0;
}

// Rotation of pair (p, q) that zeroes M[p][q] (Rutishauser's form): returns
// t (0 = no rotation), c, s with J[p][p] = J[q][q] = c, J[p][q] = s,
// J[q][p] = -s.
__device__ __forceinline__ double jacobi_angle(const double *Mc, int m, int p, int q, double &c, double &s,
                                               double &app, double &aqq, double &apq) {
  app = Mc[(int64_t)p * m + p];
  aqq = Mc[(int64_t)q * m + q];
  apq = Mc[(int64_t)p * m + q];
  c = 1.0;
  s = 0.0;
  const double aabs = fabs(apq);
  if (!(aabs > 1e-300) || aabs <= kJacobiTol * sqrt(fabs(app) * fabs(aqq))) return 0.0;
  const double theta = (aqq - app) / (2.0 * apq);
  const double t = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + hypot(1.0, theta));
  c = 1.0 / sqrt(1.0 + t * t);
  s = t * c;
  return t;
}

// Upper-triangle block t (< h(h+1)/2, row-major over a <= b) -> (a, b): a
// single-precision root (exact operands below 2^24), then integer steps.
__device__ __forceinline__ void upper_block(int h, int t, int &a, int &b) {
  const float w = 2.0f * (float)h + 1.0f;
  int x = (int)floorf((w - sqrtf(w * w - 8.0f * (float)t)) * 0.5f);
  x = x < 0 ? 0 : (x >= h ? h - 1 : x);
  auto start = [h](int r) { return r * h - r * (r - 1) / 2; };
  while (x > 0 && start(x) > t) --x;
  while (x + 1 < h && start(x + 1) <= t) ++x;
  a = x;
  b = x + (t - start(x));
}

// 3. Jacobi sweeps for every problem (cooperative launch).  M and V^T are
// [P][2][m][m]; round g reads buffer g & 1 and writes the other one.  CTA c
// owns the items [c N / G, (c+1) N / G) of the N = P (h(h+1)/2 + h m) items
// of a round (upper blocks of M, then the rotated row pairs of V^T, problem
// by problem), so it meets one or two problems per round and computes their
// h rotations once, into shared memory.
__global__ void __launch_bounds__(256) basis_jacobi_kernel(BasisShape bs, double *__restrict__ M,
                                                           double *__restrict__ V, BasisCtl *ctl) {
  __shared__ int flag_s, rot_s;
  __shared__ int ns_s[S4R_MAX_D_MODEL];            // next-round slot of the player in slot u
  __shared__ double c_s[S4R_MAX_D_MODEL / 2], s_s[S4R_MAX_D_MODEL / 2], t_s[S4R_MAX_D_MODEL / 2];
  const int m = bs.m, h = m / 2, n1 = m - 1;
  const int64_t mm = (int64_t)m * m;
  const int64_t nMp = (int64_t)h * (h + 1) / 2, nUp = nMp + (int64_t)h * m;   // items per problem
  const int64_t N = (int64_t)bs.P * nUp;
  const int64_t i_begin = N * blockIdx.x / gridDim.x, i_end = N * (blockIdx.x + 1) / gridDim.x;
  if (threadIdx.x == 0) rot_s = 0;
  uint32_t gen = 0, round = 0;
  bool converged = false;
  for (int sweep = 0; sweep < kBasisMaxSweeps && !converged; ++sweep) {
    for (int k = 0; k < n1; ++k, ++round) {
      const int cur = (int)(round & 1u);
      const int kn = (k + 1) % n1;
      for (int u = threadIdx.x; u < m; u += blockDim.x) ns_s[u] = jac_slot(m, kn, jac_player(m, k, u));
      for (int64_t p0 = i_begin / nUp; p0 * nUp < i_end; ++p0) {
        const int p = (int)p0;
        const double *Mc = M + ((int64_t)p * 2 + cur) * mm;
        double *Mn = M + ((int64_t)p * 2 + (cur ^ 1)) * mm;
        const double *Vc = V + ((int64_t)p * 2 + cur) * mm;
        double *Vn = V + ((int64_t)p * 2 + (cur ^ 1)) * mm;
        __syncthreads();   // ns_s written; the previous problem's rotations consumed
        for (int a = threadIdx.x; a < h; a += blockDim.x) {
          double c, sn, app, aqq, apq;
          const double t = jacobi_angle(Mc, m, 2 * a, 2 * a + 1, c, sn, app, aqq, apq);
          c_s[a] = c;
          s_s[a] = sn;
          t_s[a] = t;
          if (t != 0.0 && fabs(apq) > kJacobiLastSweep * sqrt(fabs(app) * fabs(aqq))) rot_s = 1;
        }
        __syncthreads();
        // Item indices within one problem stay below 2^31 (32-bit arithmetic).
        const int lo = (int)(i_begin > p0 * nUp ? i_begin - p0 * nUp : 0);
        const int hi = (int)(i_end < (p0 + 1) * nUp ? i_end - p0 * nUp : nUp);
        const int nM32 = (int)nMp;
        for (int it = lo + (int)threadIdx.x; it < hi; it += blockDim.x) {
          if (it < nM32) {
            int a, b;
            upper_block(h, it, a, b);
            const int r0 = ns_s[2 * a], r1 = ns_s[2 * a + 1];
            const double ca = c_s[a], sa = s_s[a], ta = t_s[a];
            if (a == b) {
              const double app = Mc[(int64_t)(2 * a) * m + 2 * a], aqq = Mc[(int64_t)(2 * a + 1) * m + 2 * a + 1];
              const double apq = Mc[(int64_t)(2 * a) * m + 2 * a + 1];
              double z00 = app, z01 = apq, z10 = Mc[(int64_t)(2 * a + 1) * m + 2 * a], z11 = aqq;
              if (ta != 0.0) {
                z00 = app - ta * apq;
                z11 = aqq + ta * apq;
                z01 = z10 = 0.0;
              }
              Mn[(int64_t)r0 * m + r0] = z00;
              Mn[(int64_t)r0 * m + r1] = z01;
              Mn[(int64_t)r1 * m + r0] = z10;
              Mn[(int64_t)r1 * m + r1] = z11;
            } else {
              const double cb = c_s[b], sb = s_s[b];
              const double2 x0 = *reinterpret_cast<const double2 *>(Mc + (int64_t)(2 * a) * m + 2 * b);
              const double2 x1 = *reinterpret_cast<const double2 *>(Mc + (int64_t)(2 * a + 1) * m + 2 * b);
              // y = R_a^T x, then z = y R_b, R = [[c, s], [-s, c]].
              const double y00 = ca * x0.x - sa * x1.x, y01 = ca * x0.y - sa * x1.y;
              const double y10 = sa * x0.x + ca * x1.x, y11 = sa * x0.y + ca * x1.y;
              const double z00 = y00 * cb - y01 * sb, z01 = y00 * sb + y01 * cb;
              const double z10 = y10 * cb - y11 * sb, z11 = y10 * sb + y11 * cb;
              const int c0 = ns_s[2 * b], c1 = ns_s[2 * b + 1];
              Mn[(int64_t)r0 * m + c0] = z00;
              Mn[(int64_t)r0 * m + c1] = z01;
              Mn[(int64_t)r1 * m + c0] = z10;
              Mn[(int64_t)r1 * m + c1] = z11;
              Mn[(int64_t)c0 * m + r0] = z00;
              Mn[(int64_t)c1 * m + r0] = z01;
              Mn[(int64_t)c0 * m + r1] = z10;
              Mn[(int64_t)c1 * m + r1] = z11;
            }
          } else {
            // V' = V J on the rows of V^T: rows 2a, 2a+1 (column i) into the
            // rows of their next slots.
            const int v = it - nM32;
            const int a = v / m, i = v - a * m;
            const double c = c_s[a], sn = s_s[a];
            const bool rot = t_s[a] != 0.0;
            const double v0 = Vc[(int64_t)(2 * a) * m + i], v1 = Vc[(int64_t)(2 * a + 1) * m + i];
            Vn[(int64_t)ns_s[2 * a] * m + i] = rot ? c * v0 - sn * v1 : v0;
            Vn[(int64_t)ns_s[2 * a + 1] * m + i] = rot ? sn * v0 + c * v1 : v1;
          }
        }
      }
      __syncthreads();
      if (threadIdx.x == 0 && rot_s) {
        atomicAdd(&ctl->rot[sweep], 1u);
        rot_s = 0;
      }
      if (!basis_grid_sync(ctl, ++gen, &flag_s)) return;
    }
    converged = *(volatile uint32_t *)&ctl->rot[sweep] == 0u;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    ctl->final_buf = round & 1u;
    if (!converged) set_status(&ctl->status, kDevStatusCheck);
  }
}

// 4. Order of the eigenvalues (decreasing, lower index first on ties), the
// singular values of the kept columns, and the check that the sample has
// rank r (a direction with sigma^2 <= 1e-13 of the largest is no direction).
__global__ void __launch_bounds__(1024) basis_order_kernel(BasisShape bs, const double *__restrict__ M,
                                                           int32_t *__restrict__ order, double *__restrict__ sig,
                                                           double *__restrict__ sigma_out, BasisCtl *ctl) {
  __shared__ double lam_s[S4R_MAX_D_MODEL];
  const int p = blockIdx.x, m = bs.m;
  const double *Mf = M + ((int64_t)p * 2 + ctl->final_buf) * m * m;
  for (int i = threadIdx.x; i < m; i += blockDim.x) lam_s[i] = Mf[(int64_t)i * m + i];
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    const double li = lam_s[i];
    int rank = 0;
    for (int j = 0; j < m; ++j) {
      const double lj = lam_s[j];
      rank += (lj > li) || (lj == li && j < i);
    }
    if (rank < bs.r) order[(int64_t)p * bs.r + rank] = i;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < bs.r; k += blockDim.x) {
    const int i = order[(int64_t)p * bs.r + k];
    const int i0 = order[(int64_t)p * bs.r];
    const double l = lam_s[i], l0 = lam_s[i0];
    const bool ok = l > 1e-13 * l0 && l0 > 0.0;
    if (!ok) set_status(&ctl->status, kDevStatusCheck);
    const double sv = ok ? sqrt(l) : 0.0;
    sig[(int64_t)p * bs.r + k] = sv;
    if (sigma_out) sigma_out[(int64_t)p * bs.r + k] = sv;
  }
}

// 5. Unsigned basis columns Bw[d][k].  Gram of the rows: B = A^T U / sigma,
// a 32 x 32 tile of (d, k) per CTA over the sample rows in chunks of 32;
// Gram of the columns: B[d][k] = V^T[order[k]][d].
template <typename T>
__global__ void __launch_bounds__(256) basis_columns_kernel(BasisShape bs, const T *__restrict__ states,
                                                            const int64_t *__restrict__ rows,
                                                            const double *__restrict__ inv,
                                                            const double *__restrict__ V,
                                                            const int32_t *__restrict__ order,
                                                            const double *__restrict__ sig, const BasisCtl *ctl,
                                                            double *__restrict__ Bw) {
  __shared__ double a_s[32][33], u_s[32][33];
  __shared__ int ord_s[32];
  const int p = blockIdx.z;
  const int d0 = blockIdx.y * 32, k0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int m = bs.m;
  const double *Vp = V + ((int64_t)p * 2 + ctl->final_buf) * m * m;   // V^T, rows in slot order
  if (threadIdx.x < 32) ord_s[threadIdx.x] = (k0 + threadIdx.x < bs.r) ? order[(int64_t)p * bs.r + k0 + threadIdx.x] : 0;
  __syncthreads();
  double *Bp = Bw + (int64_t)p * bs.D * bs.r;
  if (!bs.t_side) {
    for (int e = threadIdx.x; e < 32 * 32; e += blockDim.x) {
      const int dd = e >> 5, kk = e & 31;
      const int d = d0 + dd, k = k0 + kk;
      if (d < bs.D && k < bs.r) Bp[(int64_t)d * bs.r + k] = Vp[(int64_t)ord_s[kk] * m + d];
    }
    return;
  }
  const int64_t *rows_p = rows + (int64_t)p * bs.T;
  const double *inv_p = inv + (int64_t)p * bs.T;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int j0 = 0; j0 < bs.T; j0 += 32) {
    for (int e = threadIdx.x; e < 32 * 32; e += blockDim.x) {
      const int hi = e >> 5, lo = e & 31;
      a_s[lo][hi] = basis_a(bs, states, rows_p, inv_p, p, j0 + hi, d0 + lo);     // consecutive threads walk d
      u_s[lo][hi] = (j0 + lo < m && k0 + hi < bs.r) ? Vp[(int64_t)ord_s[hi] * m + j0 + lo] : 0.0;   // ... and j
    }
    __syncthreads();
#pragma unroll 8
    for (int jj = 0; jj < 32; ++jj) {
      const double uv = u_s[jj][tx];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fma(a_s[ty + 8 * q][jj], uv, acc[q]);
    }
    __syncthreads();
  }
  const int k = k0 + tx;
  if (k < bs.r) {
    const double sv = sig[(int64_t)p * bs.r + k];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int d = d0 + ty + 8 * q;
      if (d < bs.D) Bp[(int64_t)d * bs.r + k] = sv > 0.0 ? acc[q] / sv : 0.0;
    }
  }
}

// 6. Sign convention and outputs: column k of problem p is flipped so that
// its largest-magnitude entry (lowest d on ties) is positive; written in
// fp64 and/or rounded to the storage type (fp64 -> fp32 -> T, nearest even).
template <typename T>
__global__ void __launch_bounds__(256) basis_output_kernel(BasisShape bs, const double *__restrict__ Bw,
                                                           double *__restrict__ basis_f64, T *__restrict__ basis_out) {
  __shared__ double best_v[8];
  __shared__ int best_i[8];
  __shared__ double sign_s;
  const int k = blockIdx.x, p = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double *Bp = Bw + (int64_t)p * bs.D * bs.r;
  double bv = -1.0;
  int bi = 0x7fffffff;
  for (int d = threadIdx.x; d < bs.D; d += blockDim.x) {
    const double a = fabs(Bp[(int64_t)d * bs.r + k]);
    if (a > bv) { bv = a; bi = d; }   // d ascends per thread: first maximum kept
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
  }
  if (lane == 0) { best_v[warp] = bv; best_i[warp] = bi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double v = best_v[0];
    int i = best_i[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
      if (best_v[w] > v || (best_v[w] == v && best_i[w] < i)) { v = best_v[w]; i = best_i[w]; }
    sign_s = (i < bs.D && Bp[(int64_t)i * bs.r + k] < 0.0) ? -1.0 : 1.0;
  }
  __syncthreads();
  const double sg = sign_s;
  for (int d = threadIdx.x; d < bs.D; d += blockDim.x) {
    const int64_t o = ((int64_t)p * bs.D + d) * bs.r + k;
    const double x = sg * Bp[(int64_t)d * bs.r + k];
    if (basis_f64) basis_f64[o] = x;
    if (basis_out) basis_out[o] = from_f<T>((float)x);
  }
}

}  // namespace s4r
