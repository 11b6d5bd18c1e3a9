// k_score_tc.cuh -- latent relevance scoring on the tensor cores: a
// persistent, warp-specialised kernel that streams the key-coefficient cache
// once.
//
// Eqs. 8-10 of S4R (review page, major comment 2, §3.2.2):
//   z[i][row] = C_K[i] . C_Q[row] / sqrt(r),
//   score[i]  = sum_row exp(z[i][row]) / sum_i' exp(z[i'][row]).
//
// Arithmetic.  Positions lie on the MMA's M (128 per tile, one TMEM lane
// each), scoring rows on N.  C_K tiles are exact bf16, but C_Q is fp32: the
// projection kernel splits C_Q log2(e) into three bf16 terms hi + mid + lo
// (24 significant bits), stored as a 3R-row operand.  Two MMAs per k-step
// accumulate hi (N = R) into a per-tile TMEM slot and mid, lo (N = 2R) into a
// scratch region; the epilogue forms y = (lo + mid) + hi in fp32 and works in
// base 2, e = 2^y.  A tile in which some |y| exceeds 100 takes per-row
// integer offsets k = floor(max_i y) and e = 2^(y - k), so nothing overflows;
// the offsets travel with the tile's row sums (ldexp in fp64).
//
// Work.  The active tiles of every problem of the call (ceil(L_p / 128) each,
// from the device-side lengths) form one list in problem order; CTA c of the
// G-CTA cooperative grid takes tiles c, c + G, c + 2G, ...  Warp roles:
//   warp 4  TMA producer: per 64-column k-block of a tile, one 16 KB TMA load
//           into a ring of stages; per problem switch, the split C_Q operand
//           (one bulk copy per k-block) into one of one or two buffers;
//   warp 5  MMA issuer (tcgen05.mma kind::f16, M = 128);
//   warps 0-3  epilogue, one TMEM lane (position) per thread.
// Pass 1, per tile: y, e, the tile's per-row sums (a shuffle transpose-
// reduction, then four warps in a fixed order) added in fp64 to the CTA's sums
// of the problem.  After its last tile of problem p the CTA adds those sums to
// the problem's row normalisers (fp64 atomics, 16 slots per row) and arrives
// on p's counter.  The e of a CTA's first kRetained tiles of p stay in their
// TMEM slot; once all min(T_p, G) CTAs that own tiles of p have arrived, the
// epilogue forms alpha_row = 2^k / l_row (fp64) and score = sum_row alpha e
// from the slot.  Tiles of p beyond the first kRetained keep no e: pass 2
// streams them again (most recently loaded, so mostly from L2) and
// recomputes e with the same arithmetic.  Problems complete independently,
// so one problem's wait overlaps the next problem's stream.
// It also accumulates, per problem, the histogram of the candidate scores'
// leading 12 bits for the top-k kernel.
#pragma once
#include "umma.cuh"

namespace s4r {

constexpr int kStcTile = 128;
constexpr int kStcThreads = 192;       // warps 0-3 epilogue, warp 4 TMA producer, warp 5 MMA issuer
constexpr float kStcRangeLimit = 100.f;
constexpr int kStcSumSlots = 16;       // row-sum atomics spread over 16 copies per row
constexpr int kStcMaxSmem = 232448;    // 227 KB per block on sm_100
constexpr int kStcKbBytes = kStcTile * 128;   // one 64-column k-block of a tile
constexpr int kStcMaxStages = 12;
constexpr int kStcMinStages = 4;
constexpr int kStcTransient = 2;       // TMEM slots of tiles whose e is not kept
constexpr int kStcControlBytes = 6144;

template <int R>
struct StcCfg {
  static_assert(R == 32 || R == 64, "scoring rows per problem");
  static constexpr int kRetained = R == 64 ? 4 : 8;              // slots whose e is kept
  static constexpr int kSlots = kRetained + kStcTransient;
  static constexpr int kScratchCol = kSlots * R;                 // (mid, lo) accumulator columns
  static_assert(kScratchCol + 2 * R <= 512, "TMEM columns");
};

__host__ __device__ constexpr int stc_kblocks(int r) { return (r + 63) / 64; }
__host__ __device__ constexpr int stc_b_bytes(int R, int r) { return stc_kblocks(r) * 3 * R * 128; }
// Split C_Q buffers: two when at least kStcMinStages ring stages still fit.
__host__ __device__ constexpr int stc_b_buffers(int R, int r) {
  return 1024 + 2 * stc_b_bytes(R, r) + kStcMinStages * kStcKbBytes + kStcControlBytes <= kStcMaxSmem ? 2 : 1;
}
__host__ __device__ constexpr int stc_stages(int R, int r) {
  return (kStcMaxSmem - 1024 - kStcControlBytes - stc_b_buffers(R, r) * stc_b_bytes(R, r)) / kStcKbBytes >
                 kStcMaxStages
             ? kStcMaxStages
             : (kStcMaxSmem - 1024 - kStcControlBytes - stc_b_buffers(R, r) * stc_b_bytes(R, r)) / kStcKbBytes;
}
__host__ __device__ constexpr int stc_smem_bytes(int R, int r) {
  return 1024 + stc_b_buffers(R, r) * stc_b_bytes(R, r) + stc_stages(R, r) * kStcKbBytes + kStcControlBytes;
}
static_assert(stc_stages(64, 256) >= kStcMinStages && stc_smem_bytes(64, 256) <= kStcMaxSmem, "smem budget");

template <int R>
struct StcControl {
  uint64_t full[kStcMaxStages], empty[kStcMaxStages];
  uint64_t b_full[2], b_empty[2];
  uint64_t acc_full;                         // MMA -> epilogue: the tile's accumulators are complete
  uint64_t scratch_free;                     // epilogue -> MMA: (mid, lo) columns read
  uint64_t slot_free[StcCfg<R>::kSlots];     // epilogue -> MMA: the slot may be overwritten
  uint64_t mma_final;                        // every MMA of the CTA has completed (teardown)
  uint32_t tmem_base;
  int flag;
  int abort;                                 // a bounded wait gave up: every role stops
  int kofs_slot[StcCfg<R>::kRetained][R];    // per-row offsets of the tile in each kept slot
  int slot_p[StcCfg<R>::kRetained];          // problem of the tile in each kept slot
  int64_t slot_row0[StcCfg<R>::kRetained];   // its first row
  int kofs[R];                               // offsets of the tile in the epilogue
  float red[4][R];                           // per-warp partial sums / maxima
  float alpha[R];
  double inv_l[R];
  int pend[StcCfg<R>::kRetained + 1];        // problems arrived on, not yet finished (FIFO)
};
static_assert(sizeof(StcControl<64>) <= kStcControlBytes && sizeof(StcControl<32>) <= kStcControlBytes,
              "control block");

// A tile of the CTA's list.
struct StcTile {
  int p;            // problem
  int64_t row0;     // first coefficient row
  int64_t L;        // L_c of the problem
  int k, n;         // index among the CTA's tiles of p, and their number
  int T;            // tiles of p
  bool pass2;       // a second pass over a tile whose e was not kept
};

// The CTA's tiles: pass 1 visits global tiles c, c + G, ... in order; pass 2
// revisits, problem by problem, the tiles with k >= kept.  Every role walks
// the same sequence.
struct StcWalker {
  const int32_t *lengths;
  int64_t cap;
  int batch, G, c, kept;
  int pass, p, T, n, k;
  int64_t S, L, g0;

  __device__ void start(const int32_t *len, int64_t cap_, int batch_, int G_, int c_, int kept_) {
    lengths = len;
    cap = cap_;
    batch = batch_;
    G = G_;
    c = c_;
    kept = kept_;
    pass = 1;
    p = -1;
    S = 0;
    T = 0;
    n = 0;
    k = 0;
  }
  // Advance to the next problem holding tiles for this pass; false at the end.
  __device__ bool next_problem() {
    while (true) {
      S += T;
      ++p;
      T = 0;
      if (p >= batch) return false;
      const int64_t Lraw = __ldg(lengths + p);
      L = (Lraw >= 0 && Lraw <= cap) ? Lraw : 0;
      T = (int)ceil_div(L, kStcTile);
      if (T == 0) continue;
      const int64_t off = (((int64_t)c - S) % G + G) % G;
      g0 = S + off;
      n = g0 < S + T ? (int)((S + T - 1 - g0) / G) + 1 : 0;
      const int kmin = pass == 1 ? 0 : kept;
      if (n > kmin) {
        k = kmin;
        return true;
      }
    }
  }
  __device__ bool next(StcTile &t) {
    while (true) {
      if (p >= 0 && p < batch && k < n) {
        t.p = p;
        t.row0 = (g0 + (int64_t)k * G - S) * kStcTile;
        t.L = L;
        t.k = k;
        t.n = n;
        t.T = T;
        t.pass2 = pass == 2;
        ++k;
        return true;
      }
      if (next_problem()) continue;
      if (pass == 2) return false;
      pass = 2;
      p = -1;
      S = 0;
      T = 0;
    }
  }
};

// Named barrier of the four epilogue warps (barrier 1, 128 threads).
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool epi_or(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v)
      : "memory");
  return out != 0;
}

// Sums (or maxima) over the warp's 32 lanes of 32 values per lane: after the
// call lane L holds, in v[0], the reduction of every lane's v[L].
template <bool kMax>
__device__ __forceinline__ void warp_transpose_reduce32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 16, n = 32; m >= 1; m >>= 1, n >>= 1) {
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = up ? v[j] : v[j + n / 2];
      const float keep = up ? v[j + n / 2] : v[j];
      const float got = __shfl_xor_sync(0xffffffffu, send, m);
      v[j] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
}

// Arrival target of problem p's counter: every CTA that owns one of its T
// tiles (one more when the test hook makes it unreachable).
__device__ __forceinline__ uint32_t stc_target(int T, int G) {
  return (uint32_t)(T < G ? T : G) + (*reinterpret_cast<volatile uint32_t *>(&g_barrier_unreachable) ? 1u : 0u);
}

template <int R>
__global__ void __launch_bounds__(kStcThreads, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tmap_ck, Shape s, const int32_t *__restrict__ lengths,
                const unsigned char *__restrict__ cqs, float *__restrict__ scores, double *__restrict__ row_sum,
                uint32_t *__restrict__ ehist, unsigned int *__restrict__ counters, uint32_t *__restrict__ status) {
  using Cfg = StcCfg<R>;
  constexpr int kR = Cfg::kRetained;
  extern __shared__ __align__(1024) unsigned char stc_smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(stc_smem_raw) + 1023) & ~uintptr_t(1023));
  const int r = s.rank_k;
  const int nkb = stc_kblocks(r);
  const int b_bytes = stc_b_bytes(R, r);
  const int nB = stc_b_buffers(R, r);
  const int NS = stc_stages(R, r);
  unsigned char *b_op = smem;
  unsigned char *ring = smem + nB * b_bytes;
  StcControl<R> *ctl = reinterpret_cast<StcControl<R> *>(ring + NS * kStcKbBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = (int)gridDim.x, c = (int)blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->b_full[i], 1);
      mbar_init(&ctl->b_empty[i], 1);
    }
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->scratch_free, 1);
    for (int i = 0; i < Cfg::kSlots; ++i) mbar_init(&ctl->slot_free[i], 1);
    mbar_init(&ctl->mma_final, 1);
    ctl->abort = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&ctl->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      auto issue = [&](uint32_t idx, const StcTile &t, int kb) {
        const uint32_t st = idx % NS;
        mbar_arrive_expect_tx(&ctl->full[st], (uint32_t)kStcKbBytes);
        tma_load_2d(ring + st * kStcKbBytes, &tmap_ck, &ctl->full[st], kb * 64,
                    (int32_t)((int64_t)t.p * s.cache_rows + t.row0));
      };
      // The cache is a call input: the first problem's first k-blocks go out
      // before the wait for the projection kernel (which writes the split C_Q
      // operand), as far as the ring holds them.
      uint32_t pre = 0;
      int p_first = -1;
      {
        StcWalker wa;
        wa.start(lengths, s.cache_rows, s.batch, G, c, kR);
        StcTile a;
        while (pre < (uint32_t)NS && wa.next(a)) {
          if (p_first < 0) p_first = a.p;
          if (a.p != p_first) break;
          for (int kb = 0; kb < nkb && pre < (uint32_t)NS; ++kb, ++pre) issue(pre, a, kb);
        }
      }
      pdl_wait();
      pdl_trigger();
      StcWalker w;
      w.start(lengths, s.cache_rows, s.batch, G, c, kR);
      StcTile t;
      int prev_p = -1;
      uint32_t n_switch = 0, issued = 0;
      bool ok = true;
      while (ok && w.next(t)) {
        if (*reinterpret_cast<volatile int *>(&ctl->abort)) break;
        if (t.p != prev_p) {
          // The split C_Q operand of the new problem, into the buffer the MMA
          // released (its previous problem's MMAs complete).
          const int buf = (int)(n_switch % nB);
          if (n_switch >= (uint32_t)nB) ok = mbar_wait(&ctl->b_empty[buf], ((n_switch / nB) - 1) & 1, status);
          if (!ok) break;
          mbar_arrive_expect_tx(&ctl->b_full[buf], (uint32_t)b_bytes);
          const unsigned char *src = cqs + (int64_t)t.p * b_bytes;
          for (int kb = 0; kb < nkb; ++kb)
            bulk_load(b_op + buf * b_bytes + kb * (3 * R * 128), src + kb * (3 * R * 128), 3 * R * 128,
                      &ctl->b_full[buf]);
          ++n_switch;
          prev_p = t.p;
        }
        for (int kb = 0; kb < nkb && ok; ++kb, ++issued) {
          if (issued < pre) continue;   // issued before the wait
          if (issued >= (uint32_t)NS) ok = mbar_wait(&ctl->empty[issued % NS], ((issued / NS) - 1) & 1, status);
          if (ok) issue(issued, t, kb);
        }
      }
      if (!ok) atomicExch(&ctl->abort, 1);
      // Drain: every copy issued into this CTA's shared memory has landed
      // before the CTA may exit (waits on phases already complete return at once).
      const uint32_t total = issued > pre ? issued : pre;
      for (uint32_t st = 0; st < (uint32_t)NS && st < total; ++st) {
        const uint32_t last = st + ((total - 1 - st) / NS) * NS;   // last fill of stage st
        mbar_wait(&ctl->full[st], (last / NS) & 1, status);
      }
      for (uint32_t i = 0; i < (uint32_t)nB && i < n_switch; ++i) {
        const uint32_t last = i + ((n_switch - 1 - i) / nB) * nB;
        mbar_wait(&ctl->b_full[i], (last / nB) & 1, status);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      StcWalker w;
      w.start(lengths, s.cache_rows, s.batch, G, c, kR);
      StcTile t;
      int prev_p = -1;
      uint32_t n_switch = 0, used = 0, n_tile = 0, j_ret = 0, u_tr = 0;
      uint32_t b_base = 0;
      bool ok = true;
      const uint32_t idesc_hi = idesc_bf16_f32(128, R, 0, 0);
      const uint32_t idesc_ml = idesc_bf16_f32(128, 2 * R, 0, 0);
      while (ok && w.next(t)) {
        if (*reinterpret_cast<volatile int *>(&ctl->abort)) break;
        if (t.p != prev_p) {
          if (prev_p >= 0) umma_commit(&ctl->b_empty[(n_switch - 1) % nB]);   // previous operand free once done
          const int buf = (int)(n_switch % nB);
          ok = mbar_wait(&ctl->b_full[buf], (n_switch / nB) & 1, status);
          if (!ok) break;
          b_base = smem_u32(b_op + buf * b_bytes);
          ++n_switch;
          prev_p = t.p;
        }
        int slot;
        if (!t.pass2 && t.k < kR) {
          slot = (int)(j_ret % kR);
          if (j_ret >= (uint32_t)kR) ok = mbar_wait(&ctl->slot_free[slot], ((j_ret / kR) - 1) & 1, status);
          ++j_ret;
        } else {
          slot = kR + (int)(u_tr % kStcTransient);
          if (u_tr >= (uint32_t)kStcTransient)
            ok = ok && mbar_wait(&ctl->slot_free[slot], ((u_tr / kStcTransient) - 1) & 1, status);
          ++u_tr;
        }
        if (ok && n_tile >= 1) ok = mbar_wait(&ctl->scratch_free, (n_tile - 1) & 1, status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_hi = tmem + (uint32_t)(slot * R);
        const uint32_t d_ml = tmem + (uint32_t)Cfg::kScratchCol;
        for (int kb = 0; kb < nkb && ok; ++kb, ++used) {
          const uint32_t st = used % NS;
          ok = mbar_wait(&ctl->full[st], (used / NS) & 1, status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(ring + st * kStcKbBytes);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = sdesc_sw128(a_base + ks * 32, 16, 1024);
            const uint64_t bh = sdesc_sw128(b_base + kb * (3 * R * 128) + ks * 32, 16, 1024);
            const uint64_t bm = sdesc_sw128(b_base + kb * (3 * R * 128) + R * 128 + ks * 32, 16, 1024);
            const uint32_t acc = (kb | ks) ? 1u : 0u;
            umma_f16(d_hi, ad, bh, idesc_hi, acc);
            umma_f16(d_ml, ad, bm, idesc_ml, acc);
          }
          umma_commit(&ctl->empty[st]);
        }
        if (!ok) break;
        umma_commit(&ctl->acc_full);
        ++n_tile;
      }
      if (!ok) atomicExch(&ctl->abort, 1);
      // Every MMA issued has completed before TMEM is released.
      umma_commit(&ctl->mma_final);
      mbar_wait(&ctl->mma_final, 0, status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- epilogue (warps 0-3)
    pdl_wait();      // the row sums, counters and histogram were zeroed by the projection kernel
    pdl_trigger();
    const int pos = threadIdx.x;                         // TMEM lane = position within the tile
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    StcWalker w;
    w.start(lengths, s.cache_rows, s.batch, G, c, kR);
    StcTile t;
    uint32_t n_tile = 0, j_ret = 0, u_tr = 0;
    int ret_head = 0;                                    // oldest kept use not yet finished
    int n_pend = 0, pend_head = 0;                       // pending problems (FIFO in ctl->pend)
    double psum = 0.0;                                   // this CTA's sum of row `pos` (pos < R) for the current problem
    int cur_p2 = -1;                                     // problem whose inv_l is loaded (pass 2)
    bool ok = true;
    const uint32_t my_slot_sum = (uint32_t)(c % kStcSumSlots);

    // alpha_row = 2^k / l_row from the problem's finished row sums (fp64).
    auto load_inv_l = [&](int p) {
      if (pos < R) {
        double l = 0.0;
        if (pos < s.n_rows) {
          double part[kStcSumSlots];
#pragma unroll
          for (int q = 0; q < kStcSumSlots; ++q)
            part[q] = __ldcg(&row_sum[((int64_t)p * kStcSumSlots + q) * s.n_rows + pos]);
#pragma unroll
          for (int q = 0; q < kStcSumSlots; ++q) l += part[q];
        }
        ctl->inv_l[pos] = l > 0.0 ? 1.0 / l : 0.0;
      }
    };
    // Histogram of the candidates' leading score bits (kExpBins bins of the
    // problem), one atomic per distinct bin of the warp.
    auto hist_add = [&](int p, float sc, bool cand) {
      const uint32_t bin = cand ? (__float_as_uint(sc) >> kExpShift) & (kExpBins - 1) : 0xffffffffu;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (cand && lane == __ffs(peers) - 1) atomicAdd(&ehist[(int64_t)p * kExpBins + bin], (uint32_t)__popc(peers));
    };
    // Wait (bounded) until problem p's counter is complete.
    auto wait_problem = [&](int p, int T) -> bool {
      if (pos == 0) {
        const uint32_t target = stc_target(T, G);
        const long long limit = wait_limit();
        const long long t0 = clock64();
        int good = 1;
        while (true) {
          uint32_t v;
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counters + p) : "memory");
          if (v >= target) break;
          if (clock64() - t0 > limit) {
            set_status(status, kDevStatusTimeout);
            good = 0;
            break;
          }
          __nanosleep(32);
        }
        ctl->flag = good;
      }
      epi_sync();
      return ctl->flag != 0;
    };
    // Scores of every kept tile of the oldest pending problem, then its slots
    // are released.
    auto finish_oldest = [&](bool ok_p) {
      const int p = ctl->pend[pend_head % (kR + 1)];
      load_inv_l(p);
      epi_sync();
      int64_t Lp = 0;
      while (ret_head < (int)j_ret && ctl->slot_p[ret_head % kR] == p) {
        const int sl = ret_head % kR;
        if (pos < R) ctl->alpha[pos] = ok_p ? (float)ldexp(ctl->inv_l[pos], ctl->kofs_slot[sl][pos]) : 0.f;
        epi_sync();
        const int64_t row0 = ctl->slot_row0[sl];
        Lp = valid_length(__ldg(lengths + p), s.cache_rows);
        float acc = 0.f;
#pragma unroll
        for (int c32 = 0; c32 < R / 32; ++c32) {
          uint32_t ev[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(sl * R + c32 * 32), ev);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) acc = fmaf(ctl->alpha[c32 * 32 + j], __uint_as_float(ev[j]), acc);
        }
        const int64_t i = row0 + pos;
        if (i < Lp) scores[(int64_t)p * s.cache_rows + i] = acc;
        hist_add(p, acc, i < Lp - s.local_window);
        tc_fence_before();
        epi_sync();
        if (pos == 0) mbar_arrive(&ctl->slot_free[sl]);
        ++ret_head;
      }
      ++pend_head;
      --n_pend;
    };

    // Wait for and finish every pending problem, oldest first.
    auto finish_all_pending = [&]() {
      while (n_pend > 0) {
        const int p_old = ctl->pend[pend_head % (kR + 1)];
        const int64_t Lo = valid_length(__ldg(lengths + p_old), s.cache_rows);
        const bool okp = ok && wait_problem(p_old, (int)ceil_div(Lo, kStcTile));
        finish_oldest(okp);
        if (!okp) ok = false;
      }
    };

    while (w.next(t)) {
      if (*reinterpret_cast<volatile int *>(&ctl->abort)) ok = false;
      if (!ok) break;
      // Pass 2 needs every problem's normalisers.
      if (t.pass2 && cur_p2 < 0) finish_all_pending();
      const bool kept = !t.pass2 && t.k < kR;
      // A kept tile reuses the slot of the kept tile kR uses earlier, which
      // belongs to an older problem: finish problems until it is released.
      while (kept && (int)j_ret - kR >= ret_head && n_pend > 0) {
        const int p_old = ctl->pend[pend_head % (kR + 1)];
        const int64_t Lo = valid_length(__ldg(lengths + p_old), s.cache_rows);
        const bool okp = ok && wait_problem(p_old, (int)ceil_div(Lo, kStcTile));
        finish_oldest(okp);
        if (!okp) ok = false;
      }
      if (t.pass2 && t.p != cur_p2) {
        // Every problem was finished before pass 2: its normalisers are complete.
        load_inv_l(t.p);
        cur_p2 = t.p;
      }
      const int slot = kept ? (int)(j_ret % kR) : kR + (int)(u_tr % kStcTransient);
      ok = mbar_wait(&ctl->acc_full, n_tile & 1, status) && ok;
      tc_fence_after();
      // y = (lo + mid) + hi for this position's R rows
      float y[R];
      const int64_t i = t.row0 + pos;
      const bool valid = i < t.L;
#pragma unroll
      for (int c32 = 0; c32 < R / 32; ++c32) {
        uint32_t hi[32], mid[32], lo[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(slot * R + c32 * 32), hi);
        tmem_ld32(tmem + lane_base + (uint32_t)(Cfg::kScratchCol + c32 * 32), mid);
        tmem_ld32(tmem + lane_base + (uint32_t)(Cfg::kScratchCol + R + c32 * 32), lo);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          y[c32 * 32 + j] = (__uint_as_float(lo[j]) + __uint_as_float(mid[j])) + __uint_as_float(hi[j]);
      }
      // The scratch (and a transient slot) may take the next tile's MMAs.
      tc_fence_before();
      epi_sync();
      if (pos == 0) {
        mbar_arrive(&ctl->scratch_free);
        if (!kept) mbar_arrive(&ctl->slot_free[slot]);
      }
      ++n_tile;
      if (kept) ++j_ret; else ++u_tr;
      // Range check: offsets only for a tile with some |y| beyond the limit.
      float amax = 0.f;
#pragma unroll
      for (int j = 0; j < R; ++j) amax = fmaxf(amax, fabsf(y[j]));
      const bool wide = epi_or(valid && amax > kStcRangeLimit);
      if (wide) {
        // k_row = floor(max over the tile's valid positions of y_row)
#pragma unroll
        for (int c32 = 0; c32 < R / 32; ++c32) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = valid ? y[c32 * 32 + j] : -INFINITY;
          warp_transpose_reduce32<true>(v);
          ctl->red[warp][c32 * 32 + lane] = v[0];
        }
        epi_sync();
        if (pos < R) {
          const float m = fmaxf(fmaxf(ctl->red[0][pos], ctl->red[1][pos]), fmaxf(ctl->red[2][pos], ctl->red[3][pos]));
          ctl->kofs[pos] = (m == -INFINITY) ? 0 : (int)floorf(m);
        }
        epi_sync();
      } else if (pos < R) {
        ctl->kofs[pos] = 0;
      }
      if (wide) {
#pragma unroll
        for (int j = 0; j < R; ++j) y[j] = valid ? ex2_approx(y[j] - (float)ctl->kofs[j]) : 0.f;
      } else {
#pragma unroll
        for (int j = 0; j < R; ++j) y[j] = valid ? ex2_approx(y[j]) : 0.f;
      }
      // y now holds e.
      if (t.pass2) {
        // Second pass: the problem is finished; score straight from e.
        if (pos < R) ctl->alpha[pos] = (float)ldexp(ctl->inv_l[pos], ctl->kofs[pos]);
        epi_sync();
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < R; ++j) acc = fmaf(ctl->alpha[j], y[j], acc);
        if (valid) scores[(int64_t)t.p * s.cache_rows + i] = acc;
        hist_add(t.p, acc, i < t.L - s.local_window);
        epi_sync();   // alpha is rewritten by the next tile
        continue;
      }
      if (kept) {
        // Keep e in the slot (the hi columns just read), with its offsets.
#pragma unroll
        for (int c32 = 0; c32 < R / 32; ++c32) {
          uint32_t ev[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) ev[j] = __float_as_uint(y[c32 * 32 + j]);
          tmem_st32(tmem + lane_base + (uint32_t)(slot * R + c32 * 32), ev);
        }
        tmem_wait_st();
        if (pos < R) ctl->kofs_slot[slot][pos] = ctl->kofs[pos];
        if (pos == 0) {
          ctl->slot_p[slot] = t.p;
          ctl->slot_row0[slot] = t.row0;
        }
      }
      // Per-row sums of e over the tile's 128 positions: within the warp by a
      // transpose-reduction, then the four warps in order.
#pragma unroll
      for (int c32 = 0; c32 < R / 32; ++c32) {
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = y[c32 * 32 + j];
        warp_transpose_reduce32<false>(v);
        ctl->red[warp][c32 * 32 + lane] = v[0];
      }
      epi_sync();
      if (pos < R) {
        const float ts = (ctl->red[0][pos] + ctl->red[1][pos]) + (ctl->red[2][pos] + ctl->red[3][pos]);
        const int kk = ctl->kofs[pos];
        psum += kk ? ldexp((double)ts, kk) : (double)ts;
      }
      if (t.k == t.n - 1) {
        // The CTA's last tile of the problem: publish its row sums, arrive.
        if (pos < R && pos < s.n_rows)
          atomicAdd(&row_sum[((int64_t)t.p * kStcSumSlots + my_slot_sum) * s.n_rows + pos], psum);
        psum = 0.0;
        __threadfence();
        epi_sync();
        if (pos == 0) {
          atomicAdd(counters + t.p, 1u);
          ctl->pend[(pend_head + n_pend) % (kR + 1)] = t.p;
        }
        ++n_pend;
        epi_sync();
      } else {
        epi_sync();   // red[] is rewritten by the next tile
      }
      // Finish problems whose counters completed meanwhile (not blocking).
      while (n_pend > 0) {
        const int p_old = ctl->pend[pend_head % (kR + 1)];
        if (pos == 0) {
          const int64_t Lo = valid_length(__ldg(lengths + p_old), s.cache_rows);
          uint32_t v;
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counters + p_old) : "memory");
          ctl->flag = v >= stc_target((int)ceil_div(Lo, kStcTile), G) ? 1 : 0;
        }
        epi_sync();
        const bool done = ctl->flag != 0;
        epi_sync();
        if (!done) break;
        finish_oldest(true);
      }
    }
    finish_all_pending();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace s4r
