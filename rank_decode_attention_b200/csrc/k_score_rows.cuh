// k_score_rows.cuh -- latent relevance scoring on the tensor cores for many
// scoring rows (the per-head reading: R = W * H_q rows, up to 512), in two
// passes over the key-coefficient cache.
//
// Eqs. 8-10 of S4R (review page, major comment 2, §3.2.2):
//   z[i][row] = C_K[i] . C_Q[row] / sqrt(r),
//   score[i]  = sum_row exp(z[i][row]) / sum_i' exp(z[i'][row]).
//
// The arithmetic is that of the other tensor-core scoring kernels
// (k_score_tc.cuh): positions on the MMA's M (128 per tile, one TMEM lane
// each), C_Q log2(e) split into three bf16 terms hi + mid + lo taken from the
// projection kernel's operand image, y = (lo + mid) + hi in fp32, e = 2^y, and
// integer per-row offsets 2^(y - k) for a tile whose |y| exceeds 100.  What
// differs is the number of rows: 3R accumulator columns per tile do not fit
// TMEM once R > 64, so the rows go through in chunks of 64 and the e of a
// tile cannot be kept until the row normalisers are known.  Hence two
// passes, each one CTA per 128-position tile:
//   pass 1  per chunk: MMA (three N = 64 products) into one of two TMEM
//           buffers while the epilogue reduces the previous chunk (its two
//           32-row halves side by side, four warps each); per-row sums of e
//           over the tile (a transposing warp butterfly, then the four warps
//           in a fixed order) added in fp64 to the row's 16 slots;
//   finish  1 / l_row = 1 / (sum of the row's slots, fixed order);
//   pass 2  the same MMAs and e (the same offsets: the same y), and
//           score = sum over the chunks and rows of e * 2^k / l_row;
//           the level-0 histogram of the candidates' scores for the top-k.
// One thread of the ninth warp issues the TMA copy of the tile (kept for
// every chunk), the chunks' operand copies (two buffers when they fit) and
// the MMAs.
#pragma once
#include "k_score_tc.cuh"

namespace s4r {

constexpr int kSrRc = 64;           // scoring rows per chunk
constexpr int kSrHalf = 128;        // epilogue threads of one 32-row half of a chunk (4 warps, one TMEM lane quadrant each)
constexpr int kSrEpi = 2 * kSrHalf; // epilogue threads: warp w reads lane quadrant w % 4 and rows of half w / 4
constexpr int kSrThreads = kSrEpi + 32;
constexpr int kSrAccCols = 256;     // TMEM columns per accumulator buffer (hi, mid, lo at +0, +64, +128)

__host__ __device__ constexpr int sr_a_bytes(int r) { return stc_kblocks(r) * kStcTile * 128; }
__host__ __device__ constexpr int sr_b_bytes(int r) { return stc_kblocks(r) * 3 * kSrRc * 128; }   // one chunk
struct SrControl {
  uint64_t a_full, b_full[2], b_empty[2], acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int pad;
  float part[2][4][32]; // per half and warp: row sums (pass 1) or maxima (wide tiles)
  int kofs[2][32];      // per half: offsets of its current 32 rows
  float alpha[2][32];   // pass 2, per half: 2^k / l of its current 32 rows
  float sc2[kStcTile];  // pass 2: the second half's part of each position's score
  double inv_l[S4R_MAX_SCORE_ROWS];   // pass 2: 1 / l of every row
};
__host__ __device__ constexpr int sr_smem_bytes(int r, int nB) {
  return 1024 + sr_a_bytes(r) + nB * sr_b_bytes(r) + (int)((sizeof(SrControl) + 127) / 128 * 128);
}
// Operand buffers: two when they fit.
__host__ __device__ constexpr int sr_buffers(int r) { return sr_smem_bytes(r, 2) <= kStcMaxSmem ? 2 : 1; }

// Named barrier `id` over n threads, and its OR-reduction of a predicate.
__device__ __forceinline__ void sr_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ bool sr_or(int id, int n, bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return out != 0;
}

template <int PASS>
__global__ void __launch_bounds__(kSrThreads, 1)
score_rows_kernel(const __grid_constant__ CUtensorMap tmap_ck, Shape s, const int32_t *__restrict__ lengths,
                  const unsigned char *__restrict__ cqs, double *__restrict__ row_sum,
                  const double *__restrict__ inv_l, float *__restrict__ scores, uint32_t *__restrict__ ehist,
                  uint32_t *__restrict__ status) {
  extern __shared__ __align__(1024) unsigned char sr_smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(sr_smem_raw) + 1023) & ~uintptr_t(1023));
  const int r = s.rank_k, R = s.n_rows, nkb = stc_kblocks(r), nch = R / kSrRc;
  const int nB = sr_buffers(r);
  unsigned char *a_op = smem;
  unsigned char *b_op = smem + sr_a_bytes(r);
  SrControl *ctl = reinterpret_cast<SrControl *>(b_op + nB * sr_b_bytes(r));
  const int tile = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool epi = threadIdx.x < kSrEpi;
  const int64_t L = valid_length(lengths[b], s.cache_rows);
  if ((int64_t)tile * kStcTile >= L) return;   // uniform: the tile is past the problem's length
  const unsigned char *img =
      cqs + ((int64_t)(blockIdx.x % kCqsCopies) * s.batch + b) * stc_b_bytes(R, r);   // this CTA's copy
  auto load_chunk = [&](int c, int q) {
    mbar_arrive_expect_tx(&ctl->b_full[q], (uint32_t)sr_b_bytes(r));
    unsigned char *dst = b_op + q * sr_b_bytes(r);
    for (int kb = 0; kb < nkb; ++kb)
      for (int term = 0; term < 3; ++term)
        // rows term*R + 64c .. + 63 of the image's k-block: 64 contiguous
        // 128-byte rows (whole 8-row swizzle atoms)
        bulk_load(dst + (kb * 3 + term) * (kSrRc * 128),
                  img + (int64_t)kb * (3 * R * 128) + (int64_t)(term * R + c * kSrRc) * 128, kSrRc * 128,
                  &ctl->b_full[q]);
  };

  if (threadIdx.x == kSrEpi) {
    mbar_init(&ctl->a_full, 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&ctl->b_full[q], 1);
      mbar_init(&ctl->b_empty[q], 1);
      mbar_init(&ctl->acc_full[q], 1);
      mbar_init(&ctl->acc_empty[q], kSrEpi / 32);   // one arrival per epilogue warp
    }
    mbar_fence_init();
    const int32_t row0 = (int32_t)((int64_t)b * s.cache_rows + (int64_t)tile * kStcTile);
    mbar_arrive_expect_tx(&ctl->a_full, (uint32_t)sr_a_bytes(r));
    for (int kb = 0; kb < nkb; ++kb) tma_load_2d(a_op + kb * (kStcTile * 128), &tmap_ck, &ctl->a_full, kb * 64, row0);
  }
  if (warp == 0) tmem_alloc(&ctl->tmem_base, 512);
  pdl_wait();      // the operand image, the zeroed sums (and for pass 2 the normalisers) come from earlier kernels
  pdl_trigger();
  if (PASS == 2)
    for (int t = threadIdx.x; t < R; t += blockDim.x) ctl->inv_l[t] = __ldcg(inv_l + (int64_t)b * R + t);
  if (threadIdx.x == kSrEpi)
    for (int c = 0; c < nch && c < nB; ++c) load_chunk(c, c);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (threadIdx.x == kSrEpi) {
    // MMA issuer: chunk c into accumulator buffer c % 2 from operand buffer c % nB.
    const uint32_t idesc = idesc_bf16_f32(128, kSrRc, 0, 0);
    const uint32_t a_base = smem_u32(a_op);
    bool ok = mbar_wait(&ctl->a_full, 0, status);
    for (int c = 0; c < nch && ok; ++c) {
      const int q = c % nB, d = c & 1;
      ok = mbar_wait(&ctl->b_full[q], (c / nB) & 1, status);
      if (ok && c >= 2) ok = mbar_wait(&ctl->acc_empty[d], ((c / 2) - 1) & 1, status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t b_base = smem_u32(b_op + q * sr_b_bytes(r));
      for (int kb = 0; kb < nkb; ++kb) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = sdesc_sw128(a_base + kb * (kStcTile * 128) + ks * 32, 16, 1024);
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            const uint64_t bd = sdesc_sw128(b_base + (kb * 3 + term) * (kSrRc * 128) + ks * 32, 16, 1024);
            umma_f16(tmem + d * kSrAccCols + term * kSrRc, ad, bd, idesc, (kb | ks) ? 1u : 0u);
          }
        }
      }
      umma_commit(&ctl->acc_full[d]);
      umma_commit(&ctl->b_empty[q]);
      if (c + nB < nch) {
        ok = mbar_wait(&ctl->b_empty[q], (c / nB) & 1, status);
        if (ok) load_chunk(c + nB, q);
      }
    }
  } else if (epi) {
    // Warp w: TMEM lane quadrant w % 4 (positions), rows 32 h .. 32 h + 31 of
    // every 64-row chunk (h = w / 4); each half has its own named barrier.
    const int quarter = warp & 3, h = warp >> 2, bid = 1 + h;
    const int p = quarter * 32 + lane;                        // position within the tile
    const int64_t pos = (int64_t)tile * kStcTile + p;
    const bool valid = pos < L;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int slot = tile % kStcSumSlots;
    float score = 0.f;
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
      const int d = c & 1;
      const int row0 = c * kSrRc + h * 32;
      ok = mbar_wait(&ctl->acc_full[d], (c / 2) & 1, status) && ok;
      tc_fence_after();
      float y[32];
      float amax = 0.f;
      {
        uint32_t hi[32], mid[32], lo[32];
        const uint32_t col = tmem + lane_base + (uint32_t)(d * kSrAccCols + h * 32);
        tmem_ld32(col, hi);
        tmem_ld32(col + kSrRc, mid);
        tmem_ld32(col + 2 * kSrRc, lo);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          y[j] = (__uint_as_float(lo[j]) + __uint_as_float(mid[j])) + __uint_as_float(hi[j]);
          amax = fmaxf(amax, fabsf(y[j]));
        }
      }
      // This warp has read its part of the accumulator buffer.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->acc_empty[d]);
      const bool wide = sr_or(bid, kSrHalf, valid && amax > kStcRangeLimit);
      if (wide) {
        // k_row = floor(max over the tile's valid positions of y_row)
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = valid ? y[j] : -INFINITY;
        warp_transpose_reduce32<true>(v);
        ctl->part[h][quarter][lane] = v[0];
        sr_bar(bid, kSrHalf);
        if (quarter == 0) {
          const float m = fmaxf(fmaxf(ctl->part[h][0][lane], ctl->part[h][1][lane]),
                                fmaxf(ctl->part[h][2][lane], ctl->part[h][3][lane]));
          ctl->kofs[h][lane] = (m == -INFINITY) ? 0 : (int)floorf(m);
          if (PASS == 2) ctl->alpha[h][lane] = (float)ldexp(ctl->inv_l[row0 + lane], ctl->kofs[h][lane]);
        }
        sr_bar(bid, kSrHalf);
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = valid ? ex2_approx(y[j] - (float)ctl->kofs[h][j]) : 0.f;
      } else {
        if (quarter == 0) {
          ctl->kofs[h][lane] = 0;
          if (PASS == 2) ctl->alpha[h][lane] = (float)ctl->inv_l[row0 + lane];
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = valid ? ex2_approx(y[j]) : 0.f;
        sr_bar(bid, kSrHalf);
      }
      // y holds e.
      if (PASS == 1) {
        warp_transpose_reduce32<false>(y);
        ctl->part[h][quarter][lane] = y[0];
        sr_bar(bid, kSrHalf);
        if (quarter == 0) {
          const float l = (ctl->part[h][0][lane] + ctl->part[h][1][lane]) + (ctl->part[h][2][lane] + ctl->part[h][3][lane]);
          const int row = row0 + lane;
          if (row < s.n_rows && l != 0.f)
            atomicAdd(&row_sum[((int64_t)b * kStcSumSlots + slot) * R + row], ldexp((double)l, ctl->kofs[h][lane]));
        }
      } else {
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) a = fmaf(ctl->alpha[h][j], y[j], a);   // 2^k_j / l_j, formed once per row
        score += a;
      }
      sr_bar(bid, kSrHalf);   // part, kofs and alpha of this half are rewritten by the next chunk
    }
    if (PASS == 2) {
      // The two halves' parts of a position's score meet once; the write
      // needs both halves' waits to have succeeded.
      if (h == 1) ctl->sc2[p] = score;
      const bool any_bad = sr_or(3, kSrEpi, !ok);
      if (h == 0 && !any_bad) {
        score += ctl->sc2[p];
        if (valid) scores[(int64_t)b * s.cache_rows + pos] = score;
        const int64_t n_cand = L > s.local_window ? L - s.local_window : 0;
        const bool cand = pos < n_cand;
        const uint32_t bin = cand ? (uint32_t)score_bin(__float_as_uint(score), score_center(s.n_rows, L)) : 0xffffffffu;
        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
        if (cand && lane == __ffs(peers) - 1) atomicAdd(&ehist[(int64_t)b * kExpBins + bin], (uint32_t)__popc(peers));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// 1 / l_row of every problem's rows from the 16 slots of its row sums (fixed
// order), for pass 2.
__global__ void __launch_bounds__(256) score_rows_finish(Shape s, const double *__restrict__ row_sum,
                                                         double *__restrict__ inv_l) {
  pdl_wait();      // the row sums come from pass 1
  const int b = blockIdx.x, R = s.n_rows;
  for (int row = threadIdx.x; row < R; row += blockDim.x) {
    double part[kStcSumSlots];
#pragma unroll
    for (int q = 0; q < kStcSumSlots; ++q) part[q] = __ldcg(&row_sum[((int64_t)b * kStcSumSlots + q) * R + row]);
    double l = 0.0;
#pragma unroll
    for (int q = 0; q < kStcSumSlots; ++q) l += part[q];
    inv_l[(int64_t)b * R + row] = l > 0.0 ? 1.0 / l : 0.0;
  }
  pdl_trigger();
}

}  // namespace s4r
