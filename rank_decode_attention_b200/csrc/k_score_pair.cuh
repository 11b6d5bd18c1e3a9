// k_score_pair.cuh -- latent relevance scoring on the tensor cores for one
// problem whose tiles fit one resident wave: each CTA takes two 128-position
// tiles and keeps their exponentials in TMEM across one grid barrier.
//
// Eqs. 8-10 of S4R (review page, major comment 2, §3.2.2):
//   z[i][row] = C_K[i] . C_Q[row] / sqrt(r),
//   score[i]  = sum_row exp(z[i][row]) / sum_i' exp(z[i'][row]).
//
// This is the latency-bound shape of a single layer's call (L_c = 32764
// coefficient rows, 128 CTAs): with so little to stream per SM, the fixed
// costs decide, and this kernel has fewer of them than the persistent
// streamer (k_score_tc.cuh), which every other shape uses.
//
// Layout of the work: positions on the MMA's M (128 per tile, one TMEM lane
// each), scoring rows on N.  C_K tiles are exact bf16, but C_Q is fp32: it is
// split into three bf16 terms hi + mid + lo (24 significant bits) that sit
// side by side on N (N = 3R), so each term is accumulated in its own TMEM
// columns and the three are added in fp32 by the epilogue.  C_Q is scaled by
// log2(e), so the epilogue works in base 2: e = 2^y with y = z log2(e).
//
// One cooperative launch, one CTA per pair of 128-position tiles: R / 8
// epilogue warps (warp w reads TMEM lanes 32 (w % 4) .. + 31 and scoring rows
// 32 (w / 4) .. + 31) and one more warp whose first thread issues the TMA
// copies and the tcgen05.mma:
//   A. TMA both C_K tiles (before the wait for the projection kernel), then
//      bulk-copy the split C_Q operand (its shared-memory image, written by the
//      projection kernel); MMA each tile into its own 256-column TMEM region.
//   B. per tile: y = hi + mid + lo, e = 2^y (kept in TMEM), per-row sums of e
//      over the tile (fp32 partials, fixed order); one fp64 atomic per row
//      and CTA adds them to the row normalisers (16 slots per row).  A tile
//      whose |y| exceeds 100 uses integer per-row offsets 2^(y - k) instead,
//      so nothing overflows.
//   C. one bounded grid barrier.
//   D. alpha[row] = 2^k / l_row (fp64); score[i] = sum_row alpha[row] e[i][row];
//      the level-0 histogram of the candidates' scores (score_bin) for the
//      top-k kernel.
// The cache is read once.
#pragma once
#include "k_score_tc.cuh"

namespace s4r {

constexpr int kSpTiles = 2;          // tiles per CTA
constexpr int kSpTmemCols = 512;
constexpr int kSpTileCols = 256;     // TMEM columns per tile region
constexpr float kSpRangeLimit = 100.f;

__host__ __device__ constexpr int sp_a_bytes(int r) { return stc_kblocks(r) * kStcTile * 128; }
__host__ __device__ constexpr int sp_red_bytes(int R) { return kStcTile * (R + 1) * 4; }
constexpr int kSpControlBytes = 2048;
// dynamic shared memory: [B operand][A tile 0][A tile 1][reduction scratch unless aliased][control],
// plus up to 1 KB lost to aligning the start to 1024 bytes.  When the scratch
// does not fit it reuses A tile 0, which is dead once tile 0's MMAs completed.
__host__ __device__ constexpr bool sp_red_aliased(int R, int r) {
  return stc_b_bytes(R, r) + kSpTiles * sp_a_bytes(r) + sp_red_bytes(R) + kSpControlBytes + 1024 > kStcMaxSmem;
}
__host__ __device__ constexpr int sp_smem_bytes(int R, int r) {
  return stc_b_bytes(R, r) + kSpTiles * sp_a_bytes(r) + (sp_red_aliased(R, r) ? 0 : sp_red_bytes(R)) +
         1024 + kSpControlBytes;
}

struct SpControl {
  uint64_t b_full;
  uint64_t tma_full[kSpTiles][4];   // per (tile, 64-wide K-block)
  uint64_t mma_done[kSpTiles];
  uint32_t tmem_base;
  int flag;
  int kofs[kSpTiles][64];
  float alpha[kSpTiles][64];
  float tile_sum[kSpTiles][64];
};
static_assert(sizeof(SpControl) <= kSpControlBytes, "control block");
static_assert(sp_smem_bytes(64, 256) <= kStcMaxSmem && sp_smem_bytes(32, 256) <= kStcMaxSmem, "smem budget");

// Threads of the kernel for R scoring rows: 4 R / 32 epilogue warps (each 32
// TMEM lanes x 32 rows) and the TMA / MMA warp.
__host__ __device__ constexpr int sp_epi_threads(int R) { return 4 * R; }
__host__ __device__ constexpr int sp_threads(int R) { return sp_epi_threads(R) + 32; }

template <int R>
__global__ void __launch_bounds__(sp_threads(R), 1)
score_pair_kernel(const __grid_constant__ CUtensorMap tmap_ck, Shape s, const int32_t *__restrict__ lengths,
                const unsigned char *__restrict__ cqs, float *__restrict__ scores, double *__restrict__ row_sum,
                uint32_t *__restrict__ ehist, unsigned int *__restrict__ bar, uint32_t *__restrict__ status) {
  static_assert(R == 32 || R == 64, "scoring rows per CTA");
  extern __shared__ __align__(1024) unsigned char sp_smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(sp_smem_raw) + 1023) & ~uintptr_t(1023));
  const int r = s.rank_k;
  const int nkb = stc_kblocks(r);
  unsigned char *b_op = smem;
  unsigned char *a_op = smem + stc_b_bytes(R, r);
  float *red = reinterpret_cast<float *>(sp_red_aliased(R, r) ? a_op : a_op + kSpTiles * sp_a_bytes(r));
  SpControl *ctl = reinterpret_cast<SpControl *>(a_op + kSpTiles * sp_a_bytes(r) +
                                                   (sp_red_aliased(R, r) ? 0 : sp_red_bytes(R)));
  constexpr int kEpi = sp_epi_threads(R);   // epilogue threads; thread kEpi issues TMA and MMA
  const int warp = threadIdx.x >> 5;
  const bool epi = threadIdx.x < kEpi;
  const int cg = warp >> 2;                  // epilogue: scoring rows 32cg .. 32cg + 31
  const int64_t tiles_cap = ceil_div(s.cache_rows, kStcTile);
  const int64_t ctas_per_problem = ceil_div(tiles_cap, kSpTiles);
  const int b = (int)(blockIdx.x / ctas_per_problem);
  const int64_t tile0 = (blockIdx.x % ctas_per_problem) * kSpTiles;
  const int64_t Lraw = lengths[b];
  const int64_t L = (Lraw >= 0 && Lraw <= s.cache_rows) ? Lraw : 0;
  int n_tiles = 0;  // active tiles of this CTA
  for (int t = 0; t < kSpTiles; ++t)
    if ((tile0 + t) < tiles_cap && (tile0 + t) * kStcTile < L) n_tiles = t + 1;

  if (threadIdx.x == kEpi) {
    mbar_init(&ctl->b_full, 1);
    for (int t = 0; t < kSpTiles; ++t) {
      for (int kb = 0; kb < 4; ++kb) mbar_init(&ctl->tma_full[t][kb], 1);
      mbar_init(&ctl->mma_done[t], 1);
    }
    mbar_fence_init();
    // A: stream this CTA's coefficient tiles, one barrier per K-block.  No
    // kernel of a decode call writes the cache, so these copies start before
    // the wait for the projection kernel.
    for (int t = 0; t < n_tiles; ++t) {
      const int32_t row = (int32_t)((int64_t)b * s.cache_rows + (tile0 + t) * kStcTile);
      for (int kb = 0; kb < nkb; ++kb) {
        mbar_arrive_expect_tx(&ctl->tma_full[t][kb], (uint32_t)(kStcTile * 128));
        tma_load_2d(a_op + t * sp_a_bytes(r) + kb * (kStcTile * 128), &tmap_ck, &ctl->tma_full[t][kb], kb * 64, row);
      }
    }
  }
  if (warp == 0) tmem_alloc(&ctl->tmem_base, kSpTmemCols);
  // Everything below may read what the projection kernel wrote (the split
  // query operand, the zeroed row sums and barrier words).
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == kEpi) {
    // The split query operand, already in its shared-memory image.
    mbar_arrive_expect_tx(&ctl->b_full, (uint32_t)stc_b_bytes(R, r));
    const unsigned char *src = cqs + ((int64_t)(blockIdx.x % kCqsCopies) * s.batch + b) * stc_b_bytes(R, r);
    for (int kb = 0; kb < nkb; ++kb)
      bulk_load(b_op + kb * (3 * R * 128), src + kb * (3 * R * 128), 3 * R * 128, &ctl->b_full);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  bool ok = true;

  if (threadIdx.x == kEpi) {
    // MMA issuer: D_t[128 x 3R] = A_t[128 x r] . B[3R x r]^T
    const uint32_t idesc = idesc_bf16_f32(128, 3 * R, 0, 0);
    const uint32_t b_base = smem_u32(b_op);
    if (n_tiles > 0) ok = mbar_wait(&ctl->b_full, 0, status);
    for (int t = 0; t < n_tiles && ok; ++t) {
      const uint32_t a_base = smem_u32(a_op + t * sp_a_bytes(r));
      for (int kb = 0; kb < nkb && ok; ++kb) {
        ok = mbar_wait(&ctl->tma_full[t][kb], 0, status);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = sdesc_sw128(a_base + kb * (kStcTile * 128) + ks * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(b_base + kb * (3 * R * 128) + ks * 32, 16, 1024);
          umma_f16(tmem + t * kSpTileCols, ad, bd, idesc, (kb | ks) ? 1u : 0u);
        }
      }
      umma_commit(&ctl->mma_done[t]);
    }
  }
  __syncwarp();

  // B: per-tile exponentials and row sums (the epilogue warps; the TMA /
  // MMA warp only joins the barriers).
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const int p = (warp & 3) * 32 + (threadIdx.x & 31);   // position within the tile (epilogue threads)
  for (int t = 0; t < n_tiles; ++t) {
    const int64_t pos = (tile0 + t) * kStcTile + p;
    const bool valid = epi && pos < L;
    const uint32_t col0 = tmem + lane_base + t * kSpTileCols;
    float amax = 0.f;
    float ev[32];   // e of this thread's position for rows 32cg .. 32cg + 31
    if (epi) {
      ok = mbar_wait(&ctl->mma_done[t], 0, status) && ok;
      tc_fence_after();
      const int c = cg;
      uint32_t hi[32], mid[32], lo[32];
      tmem_ld32(col0 + c * 32, hi);
      tmem_ld32(col0 + R + c * 32, mid);
      tmem_ld32(col0 + 2 * R + c * 32, lo);
      tmem_wait_ld();
      uint32_t eb[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float y = (__uint_as_float(lo[j]) + __uint_as_float(mid[j])) + __uint_as_float(hi[j]);
        hi[j] = __float_as_uint(y);
        amax = valid ? fmaxf(amax, fabsf(y)) : amax;
        ev[j] = valid ? ex2_approx(y) : 0.f;
        eb[j] = __float_as_uint(ev[j]);
      }
      tmem_st32(col0 + c * 32, hi);      // y
      tmem_st32(col0 + R + c * 32, eb);  // e
      tmem_wait_st();
    }
    const bool wide = __syncthreads_or(amax > kSpRangeLimit) != 0;
    if (wide) {
      // Rare path: per-row integer offsets k = floor(max_i y) for this tile.
      const int c = cg;
      if (epi) {
        uint32_t yv[32];
        tmem_ld32(col0 + c * 32, yv);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) red[p * (R + 1) + c * 32 + j] = valid ? __uint_as_float(yv[j]) : -INFINITY;
      }
      __syncthreads();
      if (threadIdx.x < R) {
        float m = -INFINITY;
        for (int q = 0; q < kStcTile; ++q) m = fmaxf(m, red[q * (R + 1) + threadIdx.x]);
        ctl->kofs[t][threadIdx.x] = (m == -INFINITY) ? 0 : (int)floorf(m);
      }
      __syncthreads();
      if (epi) {
        uint32_t yv[32], eb[32];
        tmem_ld32(col0 + c * 32, yv);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          ev[j] = valid ? ex2_approx(__uint_as_float(yv[j]) - (float)ctl->kofs[t][c * 32 + j]) : 0.f;
          eb[j] = __float_as_uint(ev[j]);
        }
        tmem_st32(col0 + R + c * 32, eb);
        tmem_wait_st();
      }
      __syncthreads();   // the scratch is read before it takes the partial sums
    } else if (threadIdx.x < R) {
      ctl->kofs[t][threadIdx.x] = 0;
    }
    // Row sums over the tile's 128 positions.  Within a warp (32 positions)
    // by a transposing butterfly: at step w the lanes with bit w set keep the
    // upper half of their rows and add their partner's, so lane j ends with
    // the sum of row 32cg + j (a fixed order); the four warps of a column
    // group are then added in a fixed order.
    if (epi) {
      const int lane = threadIdx.x & 31;
#pragma unroll
      for (int w = 16; w >= 1; w >>= 1) {
        const bool upper = (lane & w) != 0;
#pragma unroll
        for (int j = 0; j < w; ++j) {
          const float send = upper ? ev[j] : ev[j + w];
          const float keep = upper ? ev[j + w] : ev[j];
          ev[j] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
      }
      red[(warp & 3) * R + cg * 32 + lane] = ev[0];
    }
    __syncthreads();
    if (threadIdx.x < R) {
      const int row = threadIdx.x;
      ctl->tile_sum[t][row] = (red[row] + red[R + row]) + (red[2 * R + row] + red[3 * R + row]);
    }
    __syncthreads();
  }
  // One fp64 atomic per row and CTA (both tiles belong to the same problem).
  if (threadIdx.x < R && threadIdx.x < s.n_rows && n_tiles > 0) {
    const int row = threadIdx.x;
    double l = 0.0;
    for (int t = 0; t < n_tiles; ++t) {
      const double v = (double)ctl->tile_sum[t][row];
      l += ctl->kofs[t][row] ? ldexp(v, ctl->kofs[t][row]) : v;
    }
    atomicAdd(&row_sum[((int64_t)b * kStcSumSlots + blockIdx.x % kStcSumSlots) * s.n_rows + row], l);
  }

  // C: every tile has added its row sums.
  const bool bar_ok = grid_barrier(bar, status, &ctl->flag);
  {

  // D: scores.  l_row = sum of the row's slots (fixed order), then its
  // fp32 reciprocal.
  if (threadIdx.x < R) {
    const int row = threadIdx.x;
    double l = 0.0;
    if (row < s.n_rows && bar_ok) {
      double part[kStcSumSlots];
#pragma unroll
      for (int q = 0; q < kStcSumSlots; ++q) part[q] = __ldcg(&row_sum[((int64_t)b * kStcSumSlots + q) * s.n_rows + row]);
#pragma unroll
      for (int q = 0; q < kStcSumSlots; ++q) l += part[q];
    }
    // alpha = 2^k / l in fp64 first: l itself may lie outside the fp32 range
    // when a row's logits are far from 0 (the tiles then carry offsets k).
    const double inv = (l > 0.0) ? 1.0 / l : 0.0;
    for (int t = 0; t < n_tiles; ++t) ctl->alpha[t][row] = (float)ldexp(inv, ctl->kofs[t][row]);
  }
  // Level-0 histogram of the candidate scores (rows before the local window;
  // score_bin around the mean R / L_c) for the top-k kernel: neighbouring
  // positions mostly share a bin, so each warp adds one count per distinct
  // bin straight into the problem's histogram.
  const uint32_t center = score_center(s.n_rows, L);
  uint32_t *hist = ehist + (int64_t)b * kExpBins;
  const int64_t n_cand = L > s.local_window ? L - s.local_window : 0;
  __syncthreads();   // alpha is written
  if (epi)
    for (int t = cg; t < n_tiles; t += R / 32) {
      const int64_t pos = (tile0 + t) * kStcTile + p;
      const uint32_t col0 = tmem + lane_base + t * kSpTileCols;
      float acc = 0.f;
#pragma unroll 1
      for (int c = 0; c < R / 32; ++c) {
        uint32_t ev[32];
        tmem_ld32(col0 + R + c * 32, ev);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) acc = fmaf(ctl->alpha[t][c * 32 + j], __uint_as_float(ev[j]), acc);
      }
      if (pos < L) scores[(int64_t)b * s.cache_rows + pos] = acc;
      const bool cand = pos < n_cand;
      const uint32_t bin = cand ? (uint32_t)score_bin(__float_as_uint(acc), center) : 0xffffffffu;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (cand && (threadIdx.x & 31) == __ffs(peers) - 1)
        asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(hist + bin), "r"((uint32_t)__popc(peers)) : "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kSpTmemCols);
}

}  // namespace s4r
