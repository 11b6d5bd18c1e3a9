// k_encode_tc.cuh -- encode C = S . B on the 5th-generation tensor cores.
//
// Eq. 3 of S4R (review page, "What carries the argument"): every non-sink
// token state is stored as its coefficients c = s . B.  For a prompt this is
// a dense GEMM, M = tokens, N = rank, K = D'.
//
// Persistent: one CTA per SM loops over 128-token tiles (tile = CTA, CTA +
// grid, ...) of one or two independent problems (the K and V halves of a
// prompt, each with its own basis: tiles 0 .. n_tiles - 1 are problem 0's),
// with three roles that run ahead of one another:
//   * warp 0 streams K-blocks of 64 with TMA (S tile: 128 x 64, K-major;
//     basis tile: 64 x rank, N-major; both 128-byte swizzled) through a
//     kEncStages-deep mbarrier ring, across tile boundaries;
//   * warp 1 issues tcgen05.mma (M = 128, N = rank, K = 16) into one of two
//     TMEM accumulators (tiles alternate), releasing each ring stage with
//     tcgen05.commit and announcing a finished accumulator the same way;
//   * warps 2-5 read a finished accumulator back (tcgen05.ld, one row per
//     thread; warp w reads TMEM lanes 32 (w % 4) ..), round to bf16, store,
//     and hand the accumulator back, while the next tile is already being
//     loaded and multiplied.
// Every wait is bounded; a wait that gives up sets the library status word
// and its role stops.
#pragma once
#include "umma.cuh"

namespace s4r {

constexpr int kEncStages = 4;
constexpr int kEncBM = 128, kEncBK = 64;
constexpr int kEncABytes = kEncBM * kEncBK * 2;  // 16 KB
constexpr int kEncThreads = 192;                 // TMA warp, MMA warp, 4 epilogue warps

__host__ __device__ constexpr int enc_b_bytes(int rank) { return ((rank + 63) / 64) * kEncBK * 64 * 2; }
__host__ __device__ constexpr int enc_stage_bytes(int rank) { return kEncABytes + enc_b_bytes(rank); }
// TMEM columns of one accumulator (two are allocated).
__host__ __device__ constexpr int enc_tmem_cols(int rank) { return rank <= 32 ? 32 : rank <= 64 ? 64 : rank <= 128 ? 128 : 256; }
__host__ inline size_t enc_smem_bytes(int rank) { return (size_t)kEncStages * enc_stage_bytes(rank) + 1024 + 256; }

// Outputs of the (at most two) problems of a launch.
template <typename OutT>
struct EncOut {
  OutT *C[2];
  int64_t ldc[2];
};

template <typename OutT>
__global__ void __launch_bounds__(kEncThreads, 1)
encode_tc_kernel(const __grid_constant__ CUtensorMap tmap_s0, const __grid_constant__ CUtensorMap tmap_b0,
                 const __grid_constant__ CUtensorMap tmap_s1, const __grid_constant__ CUtensorMap tmap_b1,
                 EncOut<OutT> o, int n_prob, int64_t n, int d, int r) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = enc_stage_bytes(r);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kEncStages * stage_bytes);
  uint64_t *empty = full + kEncStages;
  uint64_t *acc_full = empty + kEncStages;   // [2]
  uint64_t *acc_empty = acc_full + 2;        // [2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (d + kEncBK - 1) / kEncBK;
  const int nb = (r + 63) / 64;
  const int64_t n_tiles = (n + kEncBM - 1) / kEncBM;   // per problem
  const int64_t all_tiles = n_prob * n_tiles;
  const uint32_t acc_cols = enc_tmem_cols(r);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kEncStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);   // one arrival per epilogue warp
    }
    mbar_fence_init();
    tma_prefetch_desc(&tmap_s0);
    tma_prefetch_desc(&tmap_b0);
    if (n_prob > 1) {
      tma_prefetch_desc(&tmap_s1);
      tma_prefetch_desc(&tmap_b1);
    }
  }
  if (warp == 0) tmem_alloc(tmem_slot, 2 * acc_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (threadIdx.x == 0) {
    // TMA producer: every K-block of every tile of this CTA, in order.
    bool ok = true;
    uint32_t it = 0;
    for (int64_t tile = blockIdx.x; tile < all_tiles && ok; tile += gridDim.x) {
      const bool p1 = tile >= n_tiles;
      const CUtensorMap *ms = p1 ? &tmap_s1 : &tmap_s0;
      const CUtensorMap *mb = p1 ? &tmap_b1 : &tmap_b0;
      const int32_t m0 = (int32_t)((p1 ? tile - n_tiles : tile) * kEncBM);
      for (int kb = 0; kb < nk && ok; ++kb, ++it) {
        const int s = (int)(it % kEncStages);
        if (it >= (uint32_t)kEncStages) ok = mbar_wait(&empty[s], ((it / kEncStages) - 1) & 1, nullptr);
        if (!ok) break;
        unsigned char *a = smem + s * stage_bytes;
        unsigned char *b = a + kEncABytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
        tma_load_2d(a, ms, &full[s], kb * kEncBK, m0);
        for (int j = 0; j < nb; ++j) tma_load_2d(b + j * (kEncBK * 128), mb, &full[s], j * 64, kb * kEncBK);
      }
    }
  } else if (threadIdx.x == 32) {
    // MMA issuer: tile i of this CTA accumulates into accumulator i % 2.
    bool ok = true;
    const uint32_t idesc = idesc_bf16_f32(128, r, 0, 1);
    uint32_t it = 0, lt = 0;
    for (int64_t tile = blockIdx.x; tile < all_tiles && ok; tile += gridDim.x, ++lt) {
      const uint32_t a = lt & 1;
      if (lt >= 2) ok = mbar_wait(&acc_empty[a], ((lt / 2) - 1) & 1, nullptr);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + a * acc_cols;
      for (int kb = 0; kb < nk && ok; ++kb, ++it) {
        const int s = (int)(it % kEncStages);
        ok = mbar_wait(&full[s], (it / kEncStages) & 1, nullptr);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * stage_bytes);
        const uint32_t b_base = a_base + kEncABytes;
#pragma unroll
        for (int ks = 0; ks < kEncBK / 16; ++ks) {
          const uint64_t ad = sdesc_sw128(a_base + ks * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(b_base + ks * 2048, kEncBK * 128, 1024);
          umma_f16(d_tmem, ad, bd, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(&acc_full[a]);
    }
  } else if (warp >= 2) {
    // Epilogue: thread (quadrant, lane) owns row tile * 128 + 32 quadrant + lane.
    const int quad = warp & 3;
    bool ok = true;
    uint32_t lt = 0;
    for (int64_t tile = blockIdx.x; tile < all_tiles && ok; tile += gridDim.x, ++lt) {
      const uint32_t a = lt & 1;
      ok = mbar_wait(&acc_full[a], (lt / 2) & 1, nullptr);
      if (!ok) break;
      tc_fence_after();
      const int p = tile >= n_tiles ? 1 : 0;
      OutT *C = o.C[p];
      const int64_t ldc = o.ldc[p];
      const int64_t row = (tile - p * n_tiles) * kEncBM + quad * 32 + lane;
      for (int c0 = 0; c0 < r; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + a * acc_cols + ((uint32_t)(quad * 32) << 16) + (uint32_t)c0, v);
        tmem_wait_ld();
        if (row >= n) continue;
        OutT *dst = C + row * ldc + c0;
        const int nc = smin(32, r - c0);
        if constexpr (sizeof(OutT) == 2) {
          if (nc == 32) {
            uint32_t pw[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              pw[i] = (uint32_t)__bfloat16_as_ushort(h2.x) | ((uint32_t)__bfloat16_as_ushort(h2.y) << 16);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
              reinterpret_cast<uint4 *>(dst)[i] = make_uint4(pw[4 * i], pw[4 * i + 1], pw[4 * i + 2], pw[4 * i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nc) dst[i] = from_f<OutT>(__uint_as_float(v[i]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nc) dst[i] = __uint_as_float(v[i]);
        }
      }
      // The accumulator has been read: hand it back to the MMA issuer.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 2 * acc_cols);
}

}  // namespace s4r
