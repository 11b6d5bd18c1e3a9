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
// G-CTA cooperative grid takes chunks of K consecutive tiles, round robin.
// Warp roles (E = R / 8 epilogue warps):
//   warps 0 .. E-1  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31
//           (one position per thread) and scoring rows 32 (w / 4) .. + 31;
//   warp E  TMA producer: per 64-column k-block of a tile, one 16 KB TMA load
//           into a ring of stages; per problem switch, the split C_Q operand
//           (one bulk copy per k-block) into one of one or two buffers;
//   warp E+1  MMA issuer (tcgen05.mma kind::f16, M = 128);
//   warp E+2  counter watcher (arrivals and completions of the problems).
// Pass 1, per tile: y, e, the tile's per-row sums (a shuffle transpose-
// reduction, then the epilogue warps in a fixed order) added in fp64 to the
// CTA's sums of the problem.  After its last tile of problem p the CTA's
// counter watcher adds those sums to the problem's row normalisers (fp64 atomics, 16
// slots per row), arrives on p's counter and, once every CTA that owns tiles
// of p has arrived, forms 1 / l_row for the epilogue.  The e of a CTA's first kRetained tiles of p stay in their
// TMEM slot; once all min(T_p, G) CTAs that own tiles of p have arrived, the
// epilogue forms alpha_row = 2^k / l_row (fp64) and score = sum_row alpha e
// from the slot.  Tiles of p beyond the first kRetained keep no e: pass 2
// streams them again (most recently loaded, so mostly from L2) and
// recomputes e with the same arithmetic.  Problems complete independently,
// so one problem's wait overlaps the next problem's stream.
// It also accumulates, per problem, the level-0 histogram of the candidate
// scores (score_bin) for the top-k kernel.
#pragma once
#include "umma.cuh"

namespace s4r {

constexpr int kStcTile = 128;
constexpr float kStcRangeLimit = 100.f;
constexpr int kStcSumSlots = 16;       // row-sum atomics spread over 16 copies per row
constexpr int kStcMaxSmem = 232448;    // 227 KB per block on sm_100
constexpr int kStcKbBytes = kStcTile * 128;   // one 64-column k-block of a tile
constexpr int kStcMaxStages = 12;
constexpr int kStcMinStages = 4;
constexpr int kStcTransient = 2;       // TMEM slots of tiles whose e is not kept
constexpr int kStcControlBytes = 10240;

template <int R>
struct StcCfg {
  static_assert(R == 32 || R == 64, "scoring rows per problem");
  static constexpr int kRetained = R == 64 ? 4 : 8;              // slots whose e is kept
  static constexpr int kSlots = kRetained + kStcTransient;
  static constexpr int kScratchCol = kSlots * R;                 // (mid, lo) accumulator columns
  static_assert(kScratchCol + 2 * R <= 512, "TMEM columns");
  // Epilogue: four warps per 32 scoring rows (warp w reads TMEM lanes
  // 32 (w % 4) ...; warps w and w + 4 take rows 0-31 and 32-63).
  static constexpr int kHalves = R / 32;
  static constexpr int kEpiWarps = 4 * kHalves;
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  static constexpr int kProducer = kEpiWarps, kMma = kEpiWarps + 1, kWatcher = kEpiWarps + 2;
  static constexpr int kThreads = 32 * (kEpiWarps + 3);
};

__host__ __device__ constexpr int stc_kblocks(int r) { return (r + 63) / 64; }
__host__ __device__ constexpr int stc_b_bytes(int R, int r) { return stc_kblocks(r) * 3 * R * 128; }
// The projection kernel writes kCqsCopies identical images of the split
// C_Q operand (copy c of every problem at c * batch * stc_b_bytes): the CTAs
// of a scoring launch read copy (CTA % kCqsCopies), so the L2 lines each
// image is read from serve a quarter of the CTAs.
constexpr int kCqsCopies = 4;
// Split C_Q buffers: one, or two (the next problem's operand loads while the
// current one is in use) when at least kStcMinStages ring stages still fit.
__host__ __device__ constexpr bool stc_two_b_fit(int R, int r) {
  return 1024 + 2 * stc_b_bytes(R, r) + kStcMinStages * kStcKbBytes + kStcControlBytes <= kStcMaxSmem;
}
__host__ __device__ constexpr int stc_stages(int R, int r, int nB) {
  return (kStcMaxSmem - 1024 - kStcControlBytes - nB * stc_b_bytes(R, r)) / kStcKbBytes > kStcMaxStages
             ? kStcMaxStages
             : (kStcMaxSmem - 1024 - kStcControlBytes - nB * stc_b_bytes(R, r)) / kStcKbBytes;
}
__host__ __device__ constexpr int stc_smem_bytes(int R, int r, int nB) {
  return 1024 + nB * stc_b_bytes(R, r) + stc_stages(R, r, nB) * kStcKbBytes + kStcControlBytes;
}
static_assert(stc_stages(64, 256, 1) >= kStcMinStages && stc_smem_bytes(64, 256, 1) <= kStcMaxSmem, "smem budget");

template <int R>
struct StcControl {
  uint64_t full[kStcMaxStages], empty[kStcMaxStages];
  uint64_t b_full[2][4], b_empty[2];           // per operand buffer: each 64-column k-block landed / buffer free
  uint64_t acc_full;                         // MMA -> epilogue: the tile's accumulators are complete
  uint64_t scratch_free;                     // epilogue warps -> MMA: (mid, lo) columns read
  uint64_t slot_free[StcCfg<R>::kSlots];     // epilogue -> MMA: the slot may be overwritten
  uint64_t mma_final;                        // every MMA of the CTA has completed (teardown)
  uint32_t tmem_base;
  int flag;
  int abort;                                 // a bounded wait gave up: every role stops
  int kofs_slot[StcCfg<R>::kRetained][R];    // per-row offsets of the tile in each kept slot
  int slot_p[StcCfg<R>::kRetained];          // problem of the tile in each kept slot
  int64_t slot_row0[StcCfg<R>::kRetained];   // its first row
  int kofs[R];                               // offsets of the tile in the epilogue
  float red[2][4][R];                        // per lane quarter partial sums (two tiles in flight) / maxima
  float alpha[StcCfg<R>::kRetained][R];      // per kept slot, of the problem being finished
  float sc_part[StcCfg<R>::kHalves == 2 ? StcCfg<R>::kRetained : 1][kStcTile];   // rows 32-63's part of a score
  double inv_l[R];                           // 1 / l of the problem in pass 2
  float alpha2[R];                           // 2^k / l of the tile in pass 2
  double inv_q[StcCfg<R>::kRetained + 1][R]; // 1 / l of the problems the watcher saw complete (ring)
  int ok_q[StcCfg<R>::kRetained + 1];
  int pend[StcCfg<R>::kRetained + 1];        // problems arrived on, not yet finished (FIFO)
  int64_t pend_L[StcCfg<R>::kRetained + 1];  // and their lengths
  volatile int arrived_seq;                  // problems the epilogue has arrived on
  volatile int done_seq;                     // problems the watcher has seen complete
  int done_snap;
};
static_assert(sizeof(StcControl<64>) <= kStcControlBytes && sizeof(StcControl<32>) <= kStcControlBytes,
              "control block");

// A tile of the CTA's list.
struct StcTile {
  int p;            // problem
  int64_t row0;     // first coefficient row
  int64_t L;        // L_c of the problem
  int T;            // tiles of p
  int k;            // index among the CTA's tiles of p (in this pass)
  bool last;        // the CTA's last tile of p (pass 1)
  bool pass2;       // a second pass over a tile whose e was not kept
};

// The CTA's tiles.  The active tiles of all problems form one list in
// problem order (global tile g); chunks of K consecutive tiles go round-robin
// to the CTAs: CTA c owns chunks c, c + G, c + 2G, ...  Pass 1 visits the
// CTA's tiles in order; pass 2 revisits, problem by problem, the tiles with
// k >= kept.  Every role walks the same sequence.
struct StcWalker {
  const int32_t *lengths;
  int64_t cap;
  int batch, G, c, K, kept;
  int pass;
  int p, T, k;           // problem of the current tile, its tiles, count in this pass
  int64_t S, L;          // first global tile and length of problem p
  int64_t gc, g;         // next chunk and next global tile of this CTA
  bool have_next;        // lookahead tile present
  int64_t g_next;

  __host__ __device__ void start(const int32_t *len, int64_t cap_, int batch_, int G_, int c_, int K_, int kept_) {
    lengths = len;
    cap = cap_;
    batch = batch_;
    G = G_;
    c = c_;
    K = K_;
    kept = kept_;
    pass = 1;
    rewind();
  }
  __host__ __device__ void rewind() {
    p = -1;
    T = 0;
    S = 0;
    k = 0;
    gc = c;
    g = (int64_t)c * K;
    g_next = raw_next();
  }
  __host__ __device__ int64_t raw_next() {
    if (g >= gc * K + K) {
      gc += G;
      g = gc * K;
    }
    return g++;
  }
  // Move the problem cursor forward to the problem holding global tile gt;
  // false when gt lies past the last problem.
  __host__ __device__ bool locate(int64_t gt) {
    while (gt >= S + T) {
      S += T;
      ++p;
      T = 0;
      k = 0;
      if (p >= batch) return false;
#ifdef __CUDA_ARCH__
      const int64_t Lraw = __ldg(lengths + p);
#else
      const int64_t Lraw = lengths[p];
#endif
      L = (Lraw >= 0 && Lraw <= cap) ? Lraw : 0;
      T = (int)ceil_div(L, kStcTile);
    }
    return true;
  }
  __host__ __device__ bool next(StcTile &t) {
    while (true) {
      const int64_t gt = g_next;
      const int p_before = p;
      if (p >= batch || !locate(gt)) {
        if (pass == 2) return false;
        pass = 2;
        rewind();
        continue;
      }
      if (p != p_before) k = 0;
      g_next = raw_next();
      const int kk = k++;
      if (pass == 2 && kk < kept) continue;   // kept in pass 1
      t.p = p;
      t.row0 = (gt - S) * kStcTile;
      t.L = L;
      t.T = T;
      t.k = kk;
      t.last = g_next >= S + T;
      t.pass2 = pass == 2;
      return true;
    }
  }
};

// CTAs that own tiles of a problem whose tiles are global tiles [S, S + T):
// the chunks intersecting it, at most G.
__host__ __device__ __forceinline__ int stc_participants(int64_t S, int T, int K, int G) {
  const int64_t n = (S + T - 1) / K - S / K + 1;
  return (int)(n < G ? n : G);
}

// Named barrier of the epilogue warps (barrier 1, N threads).
template <int N>
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory"); }
template <int N>
__device__ __forceinline__ bool epi_or(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v), "n"(N)
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

// Arrival target of a problem's counter: every CTA that owns one of its
// tiles (one more when the test hook makes it unreachable).
__device__ __forceinline__ uint32_t stc_target(int participants) {
  return (uint32_t)participants + (*reinterpret_cast<volatile uint32_t *>(&g_barrier_unreachable) ? 1u : 0u);
}

template <int R>
__global__ void __launch_bounds__(StcCfg<R>::kThreads, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tmap_ck, Shape s, const int32_t *__restrict__ lengths,
                const unsigned char *__restrict__ cqs, float *__restrict__ scores, double *__restrict__ row_sum,
                uint32_t *__restrict__ ehist, unsigned int *__restrict__ counters, uint32_t *__restrict__ status,
                int K, int nB) {
  using Cfg = StcCfg<R>;
  constexpr int kR = Cfg::kRetained;
  constexpr int EN = Cfg::kEpiThreads;
  extern __shared__ __align__(1024) unsigned char stc_smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(stc_smem_raw) + 1023) & ~uintptr_t(1023));
  const int r = s.rank_k;
  const int nkb = stc_kblocks(r);
  const int b_bytes = stc_b_bytes(R, r);
  const int NS = stc_stages(R, r, nB);
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
      for (int kb = 0; kb < 4; ++kb) mbar_init(&ctl->b_full[i][kb], 1);
      mbar_init(&ctl->b_empty[i], 1);
    }
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->scratch_free, Cfg::kEpiWarps);   // one arrival per epilogue warp
    for (int i = 0; i < Cfg::kSlots; ++i) mbar_init(&ctl->slot_free[i], 1);
    mbar_init(&ctl->mma_final, 1);
    ctl->abort = 0;
    ctl->arrived_seq = 0;
    ctl->done_seq = 0;
    mbar_fence_init();
  }
  __syncthreads();
  // The cache is a call input: the first problem's first k-blocks go out
  // before the wait for the projection kernel (which writes the split C_Q
  // operand), as far as the ring holds them, and before TMEM is allocated.
  uint32_t pre = 0;
  if (warp == Cfg::kProducer && lane == 0) {
    tma_prefetch_desc(&tmap_ck);
    StcWalker wa;
    wa.start(lengths, s.cache_rows, s.batch, G, c, K, kR);
    StcTile a;
    int p_first = -1;
    while (pre < (uint32_t)NS && wa.next(a)) {
      if (p_first < 0) p_first = a.p;
      if (a.p != p_first || a.pass2) break;
      for (int kb = 0; kb < nkb && pre < (uint32_t)NS; ++kb, ++pre) {
        mbar_arrive_expect_tx(&ctl->full[pre], (uint32_t)kStcKbBytes);
        tma_load_2d(ring + pre * kStcKbBytes, &tmap_ck, &ctl->full[pre], kb * 64,
                    (int32_t)((int64_t)a.p * s.cache_rows + a.row0));
      }
    }
  }
  if (warp == 0) tmem_alloc(&ctl->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == Cfg::kProducer) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      auto issue = [&](uint32_t idx, const StcTile &t, int kb) {
        const uint32_t st = idx % NS;
        mbar_arrive_expect_tx(&ctl->full[st], (uint32_t)kStcKbBytes);
        tma_load_2d(ring + st * kStcKbBytes, &tmap_ck, &ctl->full[st], kb * 64,
                    (int32_t)((int64_t)t.p * s.cache_rows + t.row0));
      };
      pdl_wait();
      pdl_trigger();
      StcWalker w;
      w.start(lengths, s.cache_rows, s.batch, G, c, K, kR);
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
          const unsigned char *src = cqs + ((int64_t)(blockIdx.x % kCqsCopies) * s.batch + t.p) * b_bytes;
          for (int kb = 0; kb < nkb; ++kb) {
            mbar_arrive_expect_tx(&ctl->b_full[buf][kb], (uint32_t)(3 * R * 128));
            bulk_load(b_op + buf * b_bytes + kb * (3 * R * 128), src + kb * (3 * R * 128), 3 * R * 128,
                      &ctl->b_full[buf][kb]);
          }
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
        for (int kb = 0; kb < nkb; ++kb) mbar_wait(&ctl->b_full[i][kb], (last / nB) & 1, status);
      }
    }
    __syncwarp();
  } else if (warp == Cfg::kMma) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      StcWalker w;
      w.start(lengths, s.cache_rows, s.batch, G, c, K, kR);
      StcTile t;
      int prev_p = -1;
      uint32_t n_switch = 0, used = 0, n_tile = 0, j_ret = 0, u_tr = 0;
      uint32_t b_base = 0, b_buf = 0, b_par = 0;
      bool ok = true;
      const uint32_t idesc_hi = idesc_bf16_f32(128, R, 0, 0);
      const uint32_t idesc_ml = idesc_bf16_f32(128, 2 * R, 0, 0);
      while (ok && w.next(t)) {
        if (*reinterpret_cast<volatile int *>(&ctl->abort)) break;
        if (t.p != prev_p) {
          if (prev_p >= 0) umma_commit(&ctl->b_empty[(n_switch - 1) % nB]);   // previous operand free once done
          b_buf = n_switch % nB;
          b_par = (n_switch / nB) & 1;
          b_base = smem_u32(b_op + b_buf * b_bytes);
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
          ok = mbar_wait(&ctl->full[st], (used / NS) & 1, status) &&
               mbar_wait(&ctl->b_full[b_buf][kb], b_par, status);   // at once after the problem's first tile
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
  } else if (warp == Cfg::kWatcher) {
    // ------------------------------------------------------- counter watcher
    // For each problem of the CTA's list, once the epilogue has arrived on
    // it: wait (bounded) until every CTA that owns tiles of it has arrived,
    // then form 1 / l_row from its 16 row-sum slots (fp64, fixed order) into
    // the ring slot of that problem and publish its completion.  The epilogue
    // reads only shared memory.
    pdl_wait();
    constexpr int Q = kR + 1;
    const uint32_t my_slot_sum = (uint32_t)(c % kStcSumSlots);
    StcWalker w;
    w.start(lengths, s.cache_rows, s.batch, G, c, K, kR);
    StcTile t;
    int q = 0;
    bool ok = true;
    while (w.next(t) && !t.pass2) {
      if (!t.last) continue;
      // The epilogue's arrival on this problem (bounded; the epilogue may stop early).
      int good = 1;
      if (lane == 0) {
        const long long limit = wait_limit();
        const long long t0 = clock64();
        while (ctl->arrived_seq <= q) {
          if (*reinterpret_cast<volatile int *>(&ctl->abort) || clock64() - t0 > limit) { good = 0; break; }
          __nanosleep(32);
        }
      }
      good = __shfl_sync(0xffffffffu, good, 0) && ok;
      __threadfence_block();
      // This CTA's row sums into the problem's normalisers (one of 16 slots
      // per row), then the arrival.
      if (good) {
        for (int row = lane; row < R && row < s.n_rows; row += 32)
          atomicAdd(&row_sum[((int64_t)t.p * kStcSumSlots + my_slot_sum) * s.n_rows + row], ctl->inv_q[q % Q][row]);
        __threadfence();
      }
      __syncwarp();
      if (lane == 0 && good) {
        atomicAdd(counters + t.p, 1u);
        const uint32_t target = stc_target(stc_participants(w.S, t.T, K, G));
        const long long limit = wait_limit();
        const long long t1 = clock64();
        while (true) {
          uint32_t v;
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counters + t.p) : "memory");
          if (v >= target) break;
          if (*reinterpret_cast<volatile int *>(&ctl->abort) || clock64() - t1 > limit) {
            set_status(status, kDevStatusTimeout);
            good = 0;
            break;
          }
          __nanosleep(32);
        }
      }
      good = __shfl_sync(0xffffffffu, good, 0);
      for (int row = lane; row < R; row += 32) {
        double l = 0.0;
        if (good && row < s.n_rows) {
          double part[kStcSumSlots];
#pragma unroll
          for (int sl = 0; sl < kStcSumSlots; ++sl)
            part[sl] = __ldcg(&row_sum[((int64_t)t.p * kStcSumSlots + sl) * s.n_rows + row]);
#pragma unroll
          for (int sl = 0; sl < kStcSumSlots; ++sl) l += part[sl];
        }
        ctl->inv_q[q % Q][row] = l > 0.0 ? 1.0 / l : 0.0;
      }
      if (lane == 0) ctl->ok_q[q % Q] = good;
      __syncwarp();
      __threadfence_block();
      if (lane == 0) ctl->done_seq = q + 1;
      if (!good) ok = false;
      ++q;
    }
  } else if (warp < Cfg::kEpiWarps) {
    // ------------------------------------------------------- epilogue
    pdl_wait();      // the row sums, counters and histogram were zeroed by the projection kernel
    pdl_trigger();
    constexpr int Q = kR + 1;
    const int ep = threadIdx.x;                          // epilogue thread
    const int quarter = warp & 3, half = warp >> 2;
    const int pos = quarter * 32 + lane;                 // TMEM lane = position within the tile
    const int rh = half * 32;                            // this thread's rows rh .. rh+31
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    StcWalker w;
    w.start(lengths, s.cache_rows, s.batch, G, c, K, kR);
    StcTile t;
    uint32_t n_tile = 0, j_ret = 0, u_tr = 0;
    int ret_head = 0;                                    // oldest kept use not yet finished
    int n_pend = 0, pend_head = 0;                       // pending problems (FIFO in ctl->pend, index q)
    double psum = 0.0;                                   // this CTA's sum of row ep (ep < R) for the current problem
    int cur_p2 = -1;                                     // problem whose inv_l is loaded (pass 2)
    bool ok = true;

    // Level-0 histogram of the candidates' scores (score_bin around the mean
    // R / L_c), one atomic per distinct bin of the warp (warps of rows 0-31).
    auto hist_add = [&](int p, int64_t Lp, float sc, bool cand) {
      const uint32_t bin = cand ? (uint32_t)score_bin(__float_as_uint(sc), score_center(s.n_rows, Lp)) : 0xffffffffu;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (cand && lane == __ffs(peers) - 1) atomicAdd(&ehist[(int64_t)p * kExpBins + bin], (uint32_t)__popc(peers));
    };
    // Scores of every kept tile of the oldest pending problem (the watcher
    // has published its 1 / l), then its slots are released.  Each thread
    // sums its 32 rows; with two row halves, the second half's parts go
    // through shared memory to the first half's threads, which write.
    auto finish_oldest = [&]() {
      const int qq = pend_head % Q;
      const int p = ctl->pend[qq];
      const bool okp = ctl->ok_q[qq] != 0;
      const int first = ret_head;
      int n_sl = 0;
      while (first + n_sl < (int)j_ret && ctl->slot_p[(first + n_sl) % kR] == p) ++n_sl;
      if (ep < R)
        for (int u = 0; u < n_sl; ++u) {
          const int sl = (first + u) % kR;
          ctl->alpha[sl][ep] = okp ? (float)ldexp(ctl->inv_q[qq][ep], ctl->kofs_slot[sl][ep]) : 0.f;
        }
      epi_sync<EN>();
      float part[kR];
#pragma unroll
      for (int u = 0; u < kR; ++u) part[u] = 0.f;
#pragma unroll
      for (int u = 0; u < kR; ++u) {
        if (u < n_sl) {
          const int sl = (first + u) % kR;
          uint32_t ev[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(sl * R + rh), ev);
          tmem_wait_ld();
          float a = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) a = fmaf(ctl->alpha[sl][rh + j], __uint_as_float(ev[j]), a);
          part[u] = a;
          if (half == 1) ctl->sc_part[u][pos] = a;
        }
      }
      tc_fence_before();
      epi_sync<EN>();
      if (half == 0) {
        const int64_t Lp = ctl->pend_L[qq];
#pragma unroll
        for (int u = 0; u < kR; ++u) {
          if (u < n_sl) {
            const int sl = (first + u) % kR;
            const float acc = Cfg::kHalves == 2 ? part[u] + ctl->sc_part[u][pos] : part[u];
            const int64_t i = ctl->slot_row0[sl] + pos;
            if (i < Lp) scores[(int64_t)p * s.cache_rows + i] = acc;
            hist_add(p, Lp, acc, i < Lp - s.local_window);
          }
        }
      }
      if (ep == 0)
        for (int u = 0; u < n_sl; ++u) mbar_arrive(&ctl->slot_free[(first + u) % kR]);
      epi_sync<EN>();   // sc_part and alpha are rewritten by the next finish
      ret_head += n_sl;
      ++pend_head;
      --n_pend;
    };
    // Wait (bounded) until the watcher has published the oldest pending problem.
    auto wait_oldest = [&]() {
      if (ep == 0) {
        const long long limit = wait_limit();
        const long long t0 = clock64();
        while (ctl->done_seq <= pend_head) {
          if (clock64() - t0 > 2 * limit) {
            set_status(status, kDevStatusTimeout);
            ctl->ok_q[pend_head % Q] = 0;
            ctl->done_seq = pend_head + 1;   // give up on it (its scores become 0)
            break;
          }
          __nanosleep(32);
        }
      }
      epi_sync<EN>();
    };

    while (w.next(t)) {
      if (*reinterpret_cast<volatile int *>(&ctl->abort)) ok = false;
      if (!ok) break;
      if (t.pass2 && cur_p2 < 0) {
        // Pass 2 needs every problem's normalisers.
        while (n_pend > 0) {
          wait_oldest();
          finish_oldest();
        }
      }
      const bool kept = !t.pass2 && t.k < kR;
      // A kept tile reuses the slot of the kept tile kR uses earlier, which
      // belongs to an older problem: finish problems until it is released.
      while (kept && (int)j_ret - kR >= ret_head && n_pend > 0) {
        wait_oldest();
        finish_oldest();
      }
      if (t.pass2 && t.p != cur_p2) {
        // 1 / l of the problem, from its finished row sums (fp64, fixed order).
        if (ep < R) {
          double l = 0.0;
          if (ep < s.n_rows) {
            double ps[kStcSumSlots];
#pragma unroll
            for (int sl = 0; sl < kStcSumSlots; ++sl)
              ps[sl] = __ldcg(&row_sum[((int64_t)t.p * kStcSumSlots + sl) * s.n_rows + ep]);
#pragma unroll
            for (int sl = 0; sl < kStcSumSlots; ++sl) l += ps[sl];
          }
          ctl->inv_l[ep] = l > 0.0 ? 1.0 / l : 0.0;
        }
        cur_p2 = t.p;
      }
      const int slot = kept ? (int)(j_ret % kR) : kR + (int)(u_tr % kStcTransient);
      ok = mbar_wait(&ctl->acc_full, n_tile & 1, status) && ok;
      tc_fence_after();
      // y = (lo + mid) + hi for this position's rows rh .. rh+31
      float y[32];
      const int64_t i = t.row0 + pos;
      const bool valid = i < t.L;
      float amax = 0.f;
      {
        uint32_t hi[32], mid[32], lo[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(slot * R + rh), hi);
        tmem_ld32(tmem + lane_base + (uint32_t)(Cfg::kScratchCol + rh), mid);
        tmem_ld32(tmem + lane_base + (uint32_t)(Cfg::kScratchCol + R + rh), lo);
        tmem_wait_ld();
        // This warp's reads of the (mid, lo) columns are done: the next
        // tile's MMAs may overwrite them once every epilogue warp says so.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->scratch_free);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          y[j] = (__uint_as_float(lo[j]) + __uint_as_float(mid[j])) + __uint_as_float(hi[j]);
          amax = fmaxf(amax, fabsf(y[j]));
        }
      }
      // One barrier: the hi columns are read (a transient slot may take the
      // next tile's MMAs), and the range check's vote.
      tc_fence_before();
      const bool wide = epi_or<EN>(valid && amax > kStcRangeLimit);
      if (ep == 0 && !kept) mbar_arrive(&ctl->slot_free[slot]);
      ++n_tile;
      if (kept) ++j_ret; else ++u_tr;
      const int rb = (int)(n_tile & 1);   // partial-sum buffer of this tile
      if (wide) {
        // Offsets only for a tile with some |y| beyond the limit:
        // k_row = floor(max over the tile's valid positions of y_row).
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = valid ? y[j] : -INFINITY;
        warp_transpose_reduce32<true>(v);
        ctl->red[rb][quarter][rh + lane] = v[0];
        epi_sync<EN>();
        if (ep < R) {
          const float m = fmaxf(fmaxf(ctl->red[rb][0][ep], ctl->red[rb][1][ep]),
                                fmaxf(ctl->red[rb][2][ep], ctl->red[rb][3][ep]));
          ctl->kofs[ep] = (m == -INFINITY) ? 0 : (int)floorf(m);
        }
        epi_sync<EN>();
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = valid ? ex2_approx(y[j] - (float)ctl->kofs[rh + j]) : 0.f;
      } else {
        if (ep < R) ctl->kofs[ep] = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = valid ? ex2_approx(y[j]) : 0.f;
      }
      // y now holds e.
      if (t.pass2) {
        // Second pass: the problem is finished; score straight from e with
        // alpha_row = 2^k / l_row, formed once per row and tile.
        if (ep < R) ctl->alpha2[ep] = (float)ldexp(ctl->inv_l[ep], wide ? ctl->kofs[ep] : 0);
        epi_sync<EN>();
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) a = fmaf(ctl->alpha2[rh + j], y[j], a);
        if (Cfg::kHalves == 2) {
          if (half == 1) ctl->sc_part[0][pos] = a;
          epi_sync<EN>();
          if (half == 0) a += ctl->sc_part[0][pos];
        }
        if (half == 0) {
          if (valid) scores[(int64_t)t.p * s.cache_rows + i] = a;
          hist_add(t.p, t.L, a, i < t.L - s.local_window);
        }
        epi_sync<EN>();   // inv_l, alpha2 and sc_part may be rewritten for the next tile
        continue;
      }
      if (kept) {
        // Keep e in the slot (the hi columns just read), with its offsets.
        uint32_t ev[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) ev[j] = __float_as_uint(y[j]);
        tmem_st32(tmem + lane_base + (uint32_t)(slot * R + rh), ev);
        tmem_wait_st();
        if (ep < R) ctl->kofs_slot[slot][ep] = ctl->kofs[ep];
        if (ep == 0) {
          ctl->slot_p[slot] = t.p;
          ctl->slot_row0[slot] = t.row0;
        }
      }
      // Per-row sums of e over the tile's 128 positions: within the warp by a
      // transpose-reduction, then the four lane quarters in order.
      warp_transpose_reduce32<false>(y);
      ctl->red[rb][quarter][rh + lane] = y[0];
      if (ep == 0) ctl->done_snap = ctl->done_seq;   // one consistent view for every thread
      epi_sync<EN>();
      const int done_snap = ctl->done_snap;
      if (ep < R) {
        const float ts = (ctl->red[rb][0][ep] + ctl->red[rb][1][ep]) + (ctl->red[rb][2][ep] + ctl->red[rb][3][ep]);
        const int kk = ctl->kofs[ep];
        psum += kk ? ldexp((double)ts, kk) : (double)ts;
      }
      if (t.last) {
        // The CTA's last tile of the problem: its row sums go to the
        // problem's ring slot (which later holds 1 / l); the watcher adds
        // them to the row normalisers and arrives on the problem's counter.
        const int qn = pend_head + n_pend;
        if (ep < R) ctl->inv_q[qn % Q][ep] = psum;
        psum = 0.0;
        epi_sync<EN>();
        if (ep == 0) {
          ctl->pend[qn % Q] = t.p;
          ctl->pend_L[qn % Q] = t.L;
          __threadfence_block();
          ctl->arrived_seq = qn + 1;
        }
        ++n_pend;
      }
      // Finish the problems the watcher has seen complete (no waiting).
      while (n_pend > 0 && done_snap > pend_head) finish_oldest();
    }
    while (ok && n_pend > 0) {
      wait_oldest();
      finish_oldest();
    }
    if (!ok && ep == 0) atomicExch(&ctl->abort, 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace s4r
