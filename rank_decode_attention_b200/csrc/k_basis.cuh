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
// eigenvectors).  Its eigenvectors come from a two-sided block Jacobi
// method.  The Gram matrix is padded with zeros to mp = m rounded up to 32
// and its indices are cut into nb = mp / 16 blocks of 16; in each round the
// blocks meet in disjoint pairs (round-robin order, every pair of blocks
// once in nb - 1 rounds).  A round first rotates, for every pair, the
// 32 x 32 principal submatrix on its indices in shared memory by parallel
// inner rounds of 16 Rutishauser rotations (in the first round of an outer
// sweep all 31 rounds, inside each block and across the two; in the others
// the 16 across, so every index pair meets once per outer sweep), keeping
// the product Q of its rotations; then every off-diagonal
// 32 x 32 tile becomes Q_a^T M[a][c] Q_c and the eigenvector rows of the
// pair become Q_a^T V^T[a].  Matrix and eigenvectors stay in natural index
// order and are updated in place.  The phases of a round are separated by
// grid-wide barriers of one cooperative launch.  The outer sweep in which no rotation
// meets an off-diagonal entry above 1e-8 of its diagonal scale is the last
// one: its rotations leave them near their squares.
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
// Block Jacobi geometry: blocks of 16 indices; a pair of blocks (32 indices)
// is the submatrix one work item rotates in shared memory.
constexpr int kBjBlock = 16;
constexpr int kBjPair = 2 * kBjBlock;
constexpr int kBjMaxRounds = kBasisMaxSweeps * (S4R_MAX_D_MODEL / kBjBlock - 1) + 1;

struct BasisShape {
  int32_t P;         // problems
  int32_t D;         // D'
  int32_t r;         // rank
  int32_t s;         // sinks
  int32_t T;         // requested sample rows T'
  int32_t m;         // Gram dimension (even)
  int32_t mp;        // m rounded up to 32: stride of M and V^T, zero padded
  int32_t t_side;    // 1: Gram of the rows (A A^T), 0: Gram of the columns (A^T A)
  int64_t state_rows;
};

// Control words at the head of the workspace.  word 0 is the sticky status.
struct BasisCtl {
  uint32_t status;
  uint32_t bar;                   // grid barrier arrivals (monotone)
  uint32_t pad[2];
  uint32_t rot[kBasisMaxSweeps];  // CTAs that met a pair above kJacobiLastSweep in sweep i
  uint32_t vq[kBjMaxRounds];      // work tickets of the eigenvector rows of round g
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
// rounds.  Pair a is the players of slots 2a and 2a+1.
__host__ __device__ __forceinline__ int jac_player(int m, int k, int u) {
  const int n1 = m - 1, a = u >> 1;
  if ((u & 1) == 0) return a == 0 ? m - 1 : (k + a) % n1;
  return a == 0 ? k % n1 : (k - a + n1) % n1;
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
    for (int i = threadIdx.x; i < kBjMaxRounds; i += blockDim.x) ctl->vq[i] = 0u;
    if (threadIdx.x == 0) ctl->bar = 0u;
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

// 2. Gram matrix M (mp x mp, zero padded) and V^T = I.  32 x 32 output tile per CTA, four
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
  double *Mp = M + (int64_t)p * bs.mp * bs.mp;
  double *Vp = V + (int64_t)p * bs.mp * bs.mp;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty + 8 * u, j = j0 + tx;
    if (i < bs.mp && j < bs.mp) {
      Mp[(int64_t)i * bs.mp + j] = acc[u];
      Vp[(int64_t)i * bs.mp + j] = (i == j) ? 1.0 : 0.0;
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

// Rotation of pair (p, q) that zeroes S[p][q] (Rutishauser's form), S a
// symmetric matrix with row stride ld: returns t (0 = no rotation), c, s
// with J[p][p] = J[q][q] = c, J[p][q] = s, J[q][p] = -s; big tells whether
// |S[p][q]| is above kJacobiLastSweep of sqrt|S[p][p] S[q][q]|.  The tests
// compare squares, so only the angle itself takes a root:
// t = sign(theta) / (|theta| + sqrt(1 + theta^2)), theta = (a_qq - a_pp) / (2 a_pq),
// with t = 1 / (2 theta) once theta^2 would overflow.
__device__ __forceinline__ double jacobi_angle(const double *S, int ld, int p, int q, double &c, double &s,
                                               bool &big) {
  const double app = S[p * ld + p], aqq = S[q * ld + q], apq = S[p * ld + q];
  c = 1.0;
  s = 0.0;
  const double a2 = apq * apq, d2 = fabs(app * aqq);
  big = a2 > (kJacobiLastSweep * kJacobiLastSweep) * d2;
  if (!(fabs(apq) > 1e-300) || a2 <= (kJacobiTol * kJacobiTol) * d2) {
    big = false;
    return 0.0;
  }
  const double theta = (aqq - app) / (2.0 * apq);
  const double at = fabs(theta);
  double t = at < 1e150 ? 1.0 / (at + sqrt(fma(at, at, 1.0))) : 0.5 / at;
  t = theta >= 0.0 ? t : -t;
  c = rsqrt(fma(t, t, 1.0));
  s = t * c;
  return t;
}

// Shared tiles are 32 x 32 doubles with a row stride of 36: the fragment
// loads of the tensor-core products below (lanes g = lane / 4 and
// q = lane % 4 reading [8 r + g][k + q] or [k + q][8 c + g]) then fall on
// distinct banks, and rows start on 16-byte boundaries.
constexpr int kBjLd = 36;
constexpr int kBjThreads = 256;
// Inner rounds over the 16 index pairs of a submatrix (blocks I and J):
// 15 rounds inside the blocks (a round-robin of 16 on each), then 16
// rounds across them (i with 16 + (i + r) mod 16).  The rounds inside the
// blocks run in the first round of each outer sweep only, so every index
// pair still meets once per sweep; the other rounds of the sweep run the
// 16 across.
constexpr int kBjInner = 2 * kBjBlock - 1;
constexpr int kBjCross0 = kBjBlock - 1;

// Global index of local index l (< 32) of block pair a in round k with nb
// blocks: l < 16 in the block of slot 2a, the others in that of slot 2a+1.
__host__ __device__ __forceinline__ int bj_index(int nb, int k, int a, int l) {
  return jac_player(nb, k, 2 * a + (l >> 4)) * kBjBlock + (l & (kBjBlock - 1));
}

// Index pair u (< 16) of inner round kk (< 31) of a 32 x 32 submatrix whose
// first 16 local indices are block I and the others block J: rounds
// 0 .. 14 pair the indices inside the blocks (a round-robin of 16 on each,
// pairs 0-7 in I, 8-15 in J), rounds 15 .. 30 pair i in I with
// 16 + (i + r) mod 16 in J (r = kk - 15).
__host__ __device__ __forceinline__ void bj_inner_pair(int kk, int u, int &x, int &y) {
  if (kk < kBjCross0) {
    const int off = u < 8 ? 0 : kBjBlock, w = u & 7;
    x = off + jac_player(kBjBlock, kk, 2 * w);
    y = off + jac_player(kBjBlock, kk, 2 * w + 1);
  } else {
    x = u;
    y = kBjBlock + (u + kk - kBjCross0) % kBjBlock;
  }
}

// One m8n8k4 fp64 tensor-core product, {d0, d1} += a b, in the PTX
// fragment layout of that shape: lane (g, q) = (lane / 4, lane % 4) holds
// a = A[g][q], b = B[q][g] and d = D[g][2q], D[g][2q + 1].
__device__ __forceinline__ void bj_dmma(double &d0, double &d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

// Warp product of a strip of C = op(A) B (32 x 32 shared tiles, op(A) =
// A^T when TA): rows 8 rt .. 8 rt + 7, columns c0 .. c0 + 8 NT - 1, into
// acc[t] = C[8 rt + g][c0 + 8 t + 2 q + {0, 1}].
template <bool TA, int NT>
__device__ __forceinline__ void bj_strip(const double (*A)[kBjLd], const double (*B)[kBjLd], int rt, int c0,
                                         double (&acc)[NT][2]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = 0.0;
#pragma unroll
  for (int k0 = 0; k0 < kBjPair; k0 += 4) {
    const double a = TA ? A[k0 + q][8 * rt + g] : A[8 * rt + g][k0 + q];
#pragma unroll
    for (int t = 0; t < NT; ++t) bj_dmma(acc[t][0], acc[t][1], a, B[k0 + q][c0 + 8 * t + g]);
  }
}

__device__ __forceinline__ void bj_copy2(double *dst, const double *src) {
  *reinterpret_cast<double2 *>(dst) = *reinterpret_cast<const double2 *>(src);
}

// Eigenvector rows of round gv (round kv of its sweep), taken from a ticket
// counter until none is left: item (problem, pair a, 64-column strip) sets
// V^T[a][strip] = Q_a^T V^T[a][strip].  Warps 0-3 form the first 32
// columns, warps 4-7 the second.
__device__ __forceinline__ void bj_rows_items(const BasisShape &bs, double *V, const double *Qbuf, BasisCtl *ctl,
                                              int gv, int kv, double (*t0)[kBjLd], double (*t1)[kBjLd],
                                              double (*t2)[kBjLd], int (*idx_s)[kBjPair], uint32_t *tk_s) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int mp = bs.mp, nb = mp / kBjBlock, npb = nb / 2, ns = (mp / kBjPair + 1) / 2;
  const uint32_t nV = (uint32_t)(bs.P * npb * ns);
  for (;;) {
    if (tid == 0) *tk_s = atomicAdd(&ctl->vq[gv], 1u);
    __syncthreads();
    const uint32_t v = *tk_s;
    if (v >= nV) break;
    const int p = (int)(v / (uint32_t)(npb * ns)), rem = (int)(v - (uint32_t)p * (npb * ns));
    const int a = rem / ns, col0 = (rem - a * ns) * 2 * kBjPair;
    const bool two = col0 + kBjPair < mp;
    double *Vp = V + (int64_t)p * mp * mp;
    const double *Qa = Qbuf + ((int64_t)p * npb + a) * (kBjPair * kBjPair);
    if (tid < kBjPair) idx_s[0][tid] = bj_index(nb, kv, a, tid);
    __syncthreads();
    for (int e = tid; e < kBjPair * kBjPair / 2; e += blockDim.x) {
      const int i = e >> 4, j = (e & 15) * 2;
      const double *row = Vp + (int64_t)idx_s[0][i] * mp + col0 + j;
      bj_copy2(&t1[i][j], Qa + i * kBjPair + j);
      bj_copy2(&t0[i][j], row);
      if (two) bj_copy2(&t2[i][j], row + kBjPair);
    }
    __syncthreads();
    if (warp < 4 || two) {
      double acc[4][2];
      bj_strip<true, 4>(t1, warp < 4 ? t0 : t2, warp & 3, 0, acc);
      double *row = Vp + (int64_t)idx_s[0][8 * (warp & 3) + g] * mp + col0 + (warp >> 2) * kBjPair + 2 * q;
#pragma unroll
      for (int t = 0; t < 4; ++t) *reinterpret_cast<double2 *>(row + 8 * t) = make_double2(acc[t][0], acc[t][1]);
    }
    __syncthreads();   // tiles, indices and the ticket are reused
  }
}

// 3. Block Jacobi sweeps for every problem (cooperative launch).  M and V^T
// are [P][mp][mp]; Qg holds two buffers [P][mp / 32][32][32] of the pair
// rotations, round g writing buffer g & 1.  Round g (round k of its sweep):
//   phase 1, items (problem, pair a): load S = M[a][a], rotate it by its
//      inner rounds, accumulate Q_a = J_1 J_2 ..., write S back
//      into M[a][a] and Q_a; a CTA done with its items then takes the
//      eigenvector rows of round g - 1 from their ticket counter (they are
//      needed by nothing before the end);
//   grid barrier;
//   phase 2, items (problem, tile a < c): M[a][c] = Q_a^T M[a][c] Q_c on
//      the tensor cores, and its transpose into M[c][a];
//   grid barrier.
// The eigenvector rows of the last round follow the last sweep.  A 2 x 2
// block of an inner round is only read and written by the thread that owns
// it, and S is kept in its upper triangle, so it needs no second buffer.
__global__ void __launch_bounds__(kBjThreads) basis_jacobi_kernel(BasisShape bs, double *__restrict__ M,
                                                                  double *__restrict__ V, double *__restrict__ Qg,
                                                                  BasisCtl *ctl) {
  __shared__ __align__(16) double t0[kBjPair][kBjLd];
  __shared__ __align__(16) double t1[kBjPair][kBjLd];
  __shared__ __align__(16) double t2[kBjPair][kBjLd];
  __shared__ __align__(16) double t3[kBjPair][kBjLd];
  __shared__ double c_s[kBjBlock], s_s[kBjBlock], tt_s[kBjBlock];
  __shared__ unsigned char sched_s[kBjInner][kBjPair];            // index pairs of each inner round
  __shared__ unsigned char ut_s[kBjBlock * (kBjBlock + 1) / 2];   // upper (a, c) pairs of 2 x 2 blocks
  __shared__ int idx_s[2][kBjPair];
  __shared__ int flag_s;
  __shared__ uint32_t tk_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, qq = lane & 3;
  const int mp = bs.mp, nb = mp / kBjBlock, npb = nb / 2, rps = nb - 1;
  const int64_t mm = (int64_t)mp * mp;
  const int64_t qbuf = (int64_t)bs.P * npb * (kBjPair * kBjPair);
  const int nA = bs.P * npb;
  const int nMt = npb * (npb - 1) / 2, nM = bs.P * nMt;
  for (int e = tid; e < kBjInner * kBjBlock; e += blockDim.x) {
    const int kk = e / kBjBlock, u = e % kBjBlock;
    int x, y;
    bj_inner_pair(kk, u, x, y);
    sched_s[kk][2 * u] = (unsigned char)x;
    sched_s[kk][2 * u + 1] = (unsigned char)y;
  }
  if (tid < kBjBlock * (kBjBlock + 1) / 2) {
    int t = tid, a = 0;
    while (t >= kBjBlock - a) { t -= kBjBlock - a; ++a; }
    ut_s[tid] = (unsigned char)((a << 4) | (a + t));
  }
  __syncthreads();
  uint32_t gen = 0;
  int g = 0;
  bool converged = false;
  for (int sweep = 0; sweep < kBasisMaxSweeps && !converged; ++sweep) {
    for (int k = 0; k < rps; ++k, ++g) {
      double *Qcur = Qg + (g & 1) * qbuf;
      // ---- phase 1: rotate the pairs' submatrices
      const int kk0 = k == 0 ? 0 : kBjCross0;
      for (int item = blockIdx.x; item < nA; item += gridDim.x) {
        const int p = item / npb, a = item - p * npb;
        double *Mp = M + (int64_t)p * mm;
        if (tid < kBjPair) idx_s[0][tid] = bj_index(nb, k, a, tid);
        __syncthreads();
        for (int e = tid; e < kBjPair * kBjPair / 2; e += blockDim.x) {
          const int i = e >> 4, j = (e & 15) * 2;
          bj_copy2(&t0[i][j], Mp + (int64_t)idx_s[0][i] * mp + idx_s[0][j]);
          t1[i][j] = (i == j) ? 1.0 : 0.0;
          t1[i][j + 1] = (i == j + 1) ? 1.0 : 0.0;
        }
        __syncthreads();
        int big = 0;
        for (int kk = kk0; kk < kBjInner; ++kk) {
          if (tid < kBjBlock) {
            double c, sn;
            bool bg;
            // S holds its upper triangle: a pair listed as (x, y) with x > y
            // is solved as (y, x), whose theta, t and s are the negatives of
            // those of (x, y) (the same rotation J).
            const int x = sched_s[kk][2 * tid], y = sched_s[kk][2 * tid + 1];
            double t = x < y ? jacobi_angle(&t0[0][0], kBjLd, x, y, c, sn, bg)
                             : jacobi_angle(&t0[0][0], kBjLd, y, x, c, sn, bg);
            if (x > y) {
              t = -t;
              sn = -sn;
            }
            c_s[tid] = c;
            s_s[tid] = sn;
            tt_s[tid] = t;
            big |= bg ? 1 : 0;
          }
          __syncthreads();
          if (tid < kBjBlock * (kBjBlock + 1) / 2) {
            const int ab = ut_s[tid], ea = ab >> 4, ec = ab & 15;
            const int pa = sched_s[kk][2 * ea], qa = sched_s[kk][2 * ea + 1];
            // S is kept in its upper triangle: entry (i, j) lives at
            // (min, max).
            auto up = [&](int i, int j) -> double & { return i < j ? t0[i][j] : t0[j][i]; };
            if (ea == ec) {
              const double t = tt_s[ea];
              if (t != 0.0) {
                double &apq = up(pa, qa);
                t0[pa][pa] -= t * apq;
                t0[qa][qa] += t * apq;
                apq = 0.0;
              }
            } else {
              const int pc = sched_s[kk][2 * ec], qc = sched_s[kk][2 * ec + 1];
              const double ca = c_s[ea], sa = s_s[ea], cb = c_s[ec], sb = s_s[ec];
              double &e00 = up(pa, pc), &e01 = up(pa, qc), &e10 = up(qa, pc), &e11 = up(qa, qc);
              const double x00 = e00, x01 = e01, x10 = e10, x11 = e11;
              // y = R_a^T x, then z = y R_c, R = [[c, s], [-s, c]].
              const double y00 = ca * x00 - sa * x10, y01 = ca * x01 - sa * x11;
              const double y10 = sa * x00 + ca * x10, y11 = sa * x01 + ca * x11;
              e00 = y00 * cb - y01 * sb;
              e01 = y00 * sb + y01 * cb;
              e10 = y10 * cb - y11 * sb;
              e11 = y10 * sb + y11 * cb;
            }
          }
          {
            // Q = Q J on the columns of index pair e, rows i and i + 16.
            const int e = tid & 15, i = tid >> 4;
            if (tt_s[e] != 0.0) {
              const int pe = sched_s[kk][2 * e], qe = sched_s[kk][2 * e + 1];
              const double c = c_s[e], sn = s_s[e];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const double q0 = t1[i + 16 * h][pe], q1 = t1[i + 16 * h][qe];
                t1[i + 16 * h][pe] = c * q0 - sn * q1;
                t1[i + 16 * h][qe] = sn * q0 + c * q1;
              }
            }
          }
          __syncthreads();
        }
        double *Qp = Qcur + ((int64_t)p * npb + a) * (kBjPair * kBjPair);
        for (int e = tid; e < kBjPair * kBjPair / 2; e += blockDim.x) {
          const int i = e >> 4, j = (e & 15) * 2;
          const double v0 = i <= j ? t0[i][j] : t0[j][i], v1 = i <= j + 1 ? t0[i][j + 1] : t0[j + 1][i];
          *reinterpret_cast<double2 *>(Mp + (int64_t)idx_s[0][i] * mp + idx_s[0][j]) = make_double2(v0, v1);
          bj_copy2(Qp + i * kBjPair + j, &t1[i][j]);
        }
        if (__syncthreads_or(big) && tid == 0) atomicAdd(&ctl->rot[sweep], 1u);   // also frees the tiles
      }
      if (g > 0) bj_rows_items(bs, V, Qg + ((g - 1) & 1) * qbuf, ctl, g - 1, (k + rps - 1) % rps, t0, t1, t2, idx_s,
                               &tk_s);
      if (!basis_grid_sync(ctl, ++gen, &flag_s)) return;
      // ---- phase 2: rotate the off-diagonal tiles
      for (int item = blockIdx.x; item < nM; item += gridDim.x) {
        const int p = item / nMt;
        int a = 0, r = item - p * nMt;
        while (r >= npb - 1 - a) { r -= npb - 1 - a; ++a; }
        const int c = a + 1 + r;
        double *Mp = M + (int64_t)p * mm;
        const double *Qp = Qcur + (int64_t)p * npb * (kBjPair * kBjPair);
        if (tid < 2 * kBjPair) idx_s[tid >> 5][tid & 31] = bj_index(nb, k, (tid >> 5) ? c : a, tid & 31);
        __syncthreads();
        for (int e = tid; e < kBjPair * kBjPair / 2; e += blockDim.x) {
          const int i = e >> 4, j = (e & 15) * 2;
          bj_copy2(&t0[i][j], Mp + (int64_t)idx_s[0][i] * mp + idx_s[1][j]);
          bj_copy2(&t1[i][j], Qp + (int64_t)a * (kBjPair * kBjPair) + i * kBjPair + j);
          bj_copy2(&t2[i][j], Qp + (int64_t)c * (kBjPair * kBjPair) + i * kBjPair + j);
        }
        __syncthreads();
        const int rt = warp & 3, c0 = (warp >> 2) * kBjBlock;
        {
          double acc[2][2];
          bj_strip<false, 2>(t0, t2, rt, c0, acc);   // Y = X Q_c
#pragma unroll
          for (int t = 0; t < 2; ++t)
            *reinterpret_cast<double2 *>(&t3[8 * rt + gq][c0 + 8 * t + 2 * qq]) = make_double2(acc[t][0], acc[t][1]);
        }
        __syncthreads();
        {
          double acc[2][2];
          bj_strip<true, 2>(t1, t3, rt, c0, acc);    // Z = Q_a^T Y
          const int i = 8 * rt + gq;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int j = c0 + 8 * t + 2 * qq;
            *reinterpret_cast<double2 *>(Mp + (int64_t)idx_s[0][i] * mp + idx_s[1][j]) =
                make_double2(acc[t][0], acc[t][1]);
            Mp[(int64_t)idx_s[1][j] * mp + idx_s[0][i]] = acc[t][0];
            Mp[(int64_t)idx_s[1][j + 1] * mp + idx_s[0][i]] = acc[t][1];
          }
        }
        __syncthreads();   // tiles reused by the next item
      }
      if (!basis_grid_sync(ctl, ++gen, &flag_s)) return;
    }
    converged = *(volatile uint32_t *)&ctl->rot[sweep] == 0u;
  }
  if (blockIdx.x == 0 && tid == 0 && !converged) set_status(&ctl->status, kDevStatusCheck);
  if (g > 0) bj_rows_items(bs, V, Qg + ((g - 1) & 1) * qbuf, ctl, g - 1, (g - 1) % rps, t0, t1, t2, idx_s, &tk_s);
}

// 4. Order of the eigenvalues (decreasing, lower index first on ties), the
// singular values of the kept columns, and the check that the sample has
// rank r (a direction with sigma^2 <= 1e-13 of the largest is no direction).
__global__ void __launch_bounds__(1024) basis_order_kernel(BasisShape bs, const double *__restrict__ M,
                                                           int32_t *__restrict__ order, double *__restrict__ sig,
                                                           double *__restrict__ sigma_out, BasisCtl *ctl) {
  __shared__ double lam_s[S4R_MAX_D_MODEL];
  const int p = blockIdx.x, m = bs.m;
  const double *Mf = M + (int64_t)p * bs.mp * bs.mp;
  for (int i = threadIdx.x; i < m; i += blockDim.x) lam_s[i] = Mf[(int64_t)i * bs.mp + i];
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
                                                            const double *__restrict__ sig,
                                                            double *__restrict__ Bw) {
  __shared__ double a_s[32][33], u_s[32][33];
  __shared__ int ord_s[32];
  const int p = blockIdx.z;
  const int d0 = blockIdx.y * 32, k0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int m = bs.m, mp = bs.mp;
  const double *Vp = V + (int64_t)p * mp * mp;   // V^T: row i is the eigenvector of M[i][i]
  if (threadIdx.x < 32) ord_s[threadIdx.x] = (k0 + threadIdx.x < bs.r) ? order[(int64_t)p * bs.r + k0 + threadIdx.x] : 0;
  __syncthreads();
  double *Bp = Bw + (int64_t)p * bs.D * bs.r;
  if (!bs.t_side) {
    for (int e = threadIdx.x; e < 32 * 32; e += blockDim.x) {
      const int dd = e >> 5, kk = e & 31;
      const int d = d0 + dd, k = k0 + kk;
      if (d < bs.D && k < bs.r) Bp[(int64_t)d * bs.r + k] = Vp[(int64_t)ord_s[kk] * mp + d];
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
      u_s[lo][hi] = (j0 + lo < m && k0 + hi < bs.r) ? Vp[(int64_t)ord_s[hi] * mp + j0 + lo] : 0.0;   // ... and j
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
