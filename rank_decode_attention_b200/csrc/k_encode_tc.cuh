// k_encode_tc.cuh -- encode C = S . B on the 5th-generation tensor cores.
//
// Eq. 3 of S4R (review page, "What carries the argument"): every non-sink
// token state is stored as its coefficients c = s . B.  For a prompt this is
// a dense GEMM, M = tokens, N = rank, K = D'.
//
// One CTA per 128-token tile (4 warps).  Thread 0 streams K-blocks of 64 with
// TMA (S tile: 128 x 64, K-major; basis tile: 64 x rank, N-major; both
// 128-byte swizzled) through a kEncStages-deep mbarrier ring; thread 32 issues
// tcgen05.mma (M = 128, N = rank, K = 16) into a TMEM accumulator and releases
// each stage with tcgen05.commit; all four warps then read the accumulator
// back (tcgen05.ld, one row per thread), round to bf16 and store.
#pragma once
#include "umma.cuh"

namespace s4r {

constexpr int kEncStages = 4;
constexpr int kEncBM = 128, kEncBK = 64;
constexpr int kEncABytes = kEncBM * kEncBK * 2;  // 16 KB

__host__ __device__ constexpr int enc_b_bytes(int rank) { return ((rank + 63) / 64) * kEncBK * 64 * 2; }
__host__ __device__ constexpr int enc_stage_bytes(int rank) { return kEncABytes + enc_b_bytes(rank); }
__host__ __device__ constexpr int enc_tmem_cols(int rank) { return rank <= 32 ? 32 : rank <= 64 ? 64 : rank <= 128 ? 128 : 256; }
__host__ inline size_t enc_smem_bytes(int rank) { return (size_t)kEncStages * enc_stage_bytes(rank) + 1024 + 256; }

template <typename OutT>
__global__ void __launch_bounds__(128, 1)
encode_tc_kernel(const __grid_constant__ CUtensorMap tmap_s, const __grid_constant__ CUtensorMap tmap_b,
                 OutT *__restrict__ C, int64_t ldc, int64_t n, int d, int r) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = enc_stage_bytes(r);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kEncStages * stage_bytes);
  uint64_t *empty = full + kEncStages;
  uint64_t *done = empty + kEncStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kEncBM;
  const int nk = (d + kEncBK - 1) / kEncBK;
  const int nb = (r + 63) / 64;
  const uint32_t tmem_cols = enc_tmem_cols(r);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kEncStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    mbar_fence_init();
    tma_prefetch_desc(&tmap_s);
    tma_prefetch_desc(&tmap_b);
  }
  if (warp == 0) tmem_alloc(tmem_slot, tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (threadIdx.x == 0) {
    // TMA producer
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % kEncStages;
      if (kb >= kEncStages) ok = mbar_wait(&empty[s], ((kb / kEncStages) - 1) & 1, nullptr);
      if (!ok) break;
      unsigned char *a = smem + s * stage_bytes;
      unsigned char *b = a + kEncABytes;
      mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
      tma_load_2d(a, &tmap_s, &full[s], kb * kEncBK, (int32_t)m0);
      for (int j = 0; j < nb; ++j) tma_load_2d(b + j * (kEncBK * 128), &tmap_b, &full[s], j * 64, kb * kEncBK);
    }
  } else if (threadIdx.x == 32) {
    // MMA issuer
    const uint32_t idesc = idesc_bf16_f32(128, r, 0, 1);
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % kEncStages;
      ok = mbar_wait(&full[s], (kb / kEncStages) & 1, nullptr);
      if (!ok) break;
      tc_fence_after();
      const uint32_t a_base = smem_u32(smem + s * stage_bytes);
      const uint32_t b_base = a_base + kEncABytes;
#pragma unroll
      for (int ks = 0; ks < kEncBK / 16; ++ks) {
        const uint64_t ad = sdesc_sw128(a_base + ks * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(b_base + ks * 2048, kEncBK * 128, 1024);
        umma_f16(tmem, ad, bd, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(&empty[s]);
    }
    umma_commit(done);
  }
  __syncwarp();
  // Epilogue: every thread owns one output row.
  ok = mbar_wait(done, 0, nullptr);
  tc_fence_after();
  const int64_t row = m0 + warp * 32 + lane;
  for (int c0 = 0; c0 < r; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
    tmem_wait_ld();
    if (!ok || row >= n) continue;
    OutT *dst = C + row * ldc + c0;
    const int nc = smin(32, r - c0);
    if constexpr (sizeof(OutT) == 2) {
      if (nc == 32) {
        uint4 pk[4];
        uint32_t *pw = reinterpret_cast<uint32_t *>(pk);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          pw[i] = *reinterpret_cast<const uint32_t *>(&h2);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) reinterpret_cast<uint4 *>(dst)[i] = pk[i];
      } else {
        for (int i = 0; i < nc; ++i) dst[i] = from_f<OutT>(__uint_as_float(v[i]));
      }
    } else {
      for (int i = 0; i < nc; ++i) dst[i] = __uint_as_float(v[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
}

}  // namespace s4r
