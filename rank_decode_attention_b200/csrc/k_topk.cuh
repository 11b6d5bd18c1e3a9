// k_topk.cuh -- selection of the top-k global positions.
//
// Eqs. 13-15 of S4R (review page, "Core claim"): the local window is always
// kept and the top-k positions among the earlier rows are added.  Candidates
// are coefficient rows 0 .. L_c-w-1; larger score first, equal scores go to
// the lower position, so the chosen set is unique.  Output: absolute
// positions n_sink + i in ascending order, -1 padded to top_k entries.
//
// Scores are non-negative floats, so their IEEE bit patterns order like the
// values.  One CTA per problem runs an 8-bit-digit radix select for the
// threshold key tau (4 histogram passes), then a stable compaction in index
// order takes every key > tau and the lowest-index keys == tau.
#pragma once
#include "common.cuh"
#include "umma.cuh"

namespace s4r {

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ int64_t valid_length(int64_t L, int64_t cap) {
  return (L >= 0 && L <= cap) ? L : 0;
}

// Pooling of candidate scores, stride 1, same padding, odd kernel: the
// largest (S4R_POOL_MAX) or the mean (S4R_POOL_AVG) of the neighbours inside
// the candidates.  The mean sums in position order in fp32 and divides by the
// count of in-range neighbours.
__global__ void pool_kernel(Shape s, const int32_t *__restrict__ lengths,
                            const float *__restrict__ scores, float *__restrict__ pooled) {
  pdl_wait();      // scores come from the preceding kernel
  pdl_trigger();
  const int b = blockIdx.y;
  const int64_t L = valid_length(lengths[b], s.cache_rows);
  const int64_t nc = n_candidates(L, s.local_window);
  const int half = s.pool_kernel / 2;
  const bool avg = s.pool_mode == S4R_POOL_AVG;
  const float *sb = scores + (int64_t)b * s.cache_rows;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nc;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j0 = smax<int64_t>(0, i - half), j1 = smin<int64_t>(nc - 1, i + half);
    float m = sb[i], sum = 0.f;
    for (int64_t j = j0; j <= j1; ++j) {
      const float v = sb[j];
      m = fmaxf(m, v);
      sum += v;
    }
    pooled[(int64_t)b * s.cache_rows + i] = avg ? sum / (float)(j1 - j0 + 1) : m;
  }
}

// Exclusive block scan of one value per thread (any multiple of 32 threads,
// at most 1024); *total receives the block total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *warp_tot, uint32_t *total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t t = (lane < (int)(blockDim.x >> 5)) ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;  // inclusive prefix of warp totals
    if (lane == 31) *total = t;
  }
  __syncthreads();
  const uint32_t before = (wid > 0 ? warp_tot[wid - 1] : 0u) + x - v;
  __syncthreads();
  return before;
}

constexpr int kTopkSmemKeys = 32768;  // keys staged in shared memory (128 KB) when they fit
// Staged key i lives at word i + i/32: a thread walking its own contiguous
// chunk of 32 keys then never shares a bank with the other lanes of its warp.
__host__ __device__ __forceinline__ int kpad(int i) { return i + (i >> 5); }
constexpr int kTopkBins = 256;         // 8-bit digits
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSample = 256;       // sampled keys that bracket the threshold
constexpr int kTopkSeg = 256;          // in-bracket candidates kept per warp
constexpr int kTopkCand = kTopkWarps * kTopkSeg;
__host__ inline size_t topk_smem_bytes(int64_t cache_rows) {
  return sizeof(uint32_t) * ((size_t)kpad(smin<int64_t>(cache_rows, kTopkSmemKeys)) + 1 + kTopkCand);
}

struct TopkShared {
  uint32_t whist[kTopkWarps][kTopkBins];
  uint32_t hist[kTopkBins];
  uint32_t sample[kTopkSample];
  uint32_t seg_count[kTopkWarps];
  uint32_t seg_above[kTopkWarps];
  uint32_t warp_tot[32];
  uint32_t total, digit, above, t_hi, t_lo, cmin, cmax;
};

template <bool kShared>
__device__ __forceinline__ uint32_t key_at(const uint32_t *keys, int i) {
  return kShared ? keys[kpad(i)] : __ldcg(keys + i);
}

// One radix pass: histogram of digit (v >> shift) & 255 over the values that
// match `prefix` under `mask`, then the digit holding the `remaining`-th
// largest.  `value(i)` returns (valid, v) for slot i < n_slots.
template <typename ValueFn>
__device__ __forceinline__ void radix_pass(ValueFn value, int n_slots, int shift, uint32_t mask, uint32_t &prefix,
                           uint32_t &remaining, TopkShared &sh) {
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < kTopkBins / 32; ++j) sh.whist[wid][lane + 32 * j] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n_slots; i += blockDim.x) {
    bool ok;
    const uint32_t v = value(i, ok);
    if (ok && (v & mask) == prefix) atomicAdd(&sh.whist[wid][(v >> shift) & 255u], 1u);
  }
  __syncthreads();
  if (threadIdx.x < kTopkBins) {
    uint32_t c = 0;
#pragma unroll 8
    for (int w = 0; w < kTopkWarps; ++w) c += sh.whist[w][threadIdx.x];
    sh.hist[threadIdx.x] = c;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t cnt[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) { cnt[j] = sh.hist[255 - (lane * 8 + j)]; sum += cnt[j]; }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    uint32_t run = incl - sum;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (run < remaining && run + cnt[j] >= remaining) {
        sh.digit = 255u - (uint32_t)(lane * 8 + j);
        sh.above = run;
      }
      run += cnt[j];
    }
  }
  __syncthreads();
  remaining -= sh.above;
  prefix |= sh.digit << shift;
  __syncthreads();
}

// Exact radix select of the need-th largest value; passes start below the
// leading bits that every value shares (known from lo_all/hi_all, the
// minimum and maximum).  Returns tau and how many values equal to tau are in
// the top `need`.
template <typename ValueFn>
__device__ __forceinline__ void radix_select(ValueFn value, int n_slots, uint32_t need, uint32_t lo_all, uint32_t hi_all,
                             TopkShared &sh, uint32_t *tau, uint32_t *take_eq) {
  const uint32_t diff = lo_all ^ hi_all;
  int top = 31;
  while (top >= 0 && !((diff >> top) & 1u)) --top;  // highest differing bit, -1 if all equal
  uint32_t prefix = 0, mask = 0, remaining = need;
  if (top < 31) {
    const uint32_t common = (top < 0) ? 0xffffffffu : ~((2u << top) - 1u);
    prefix = lo_all & common;
    mask = common;
  }
  if (top >= 0) {
    // digits whose 8-bit window covers bits top..0, aligned to multiples of 8
    for (int shift = (top / 8) * 8; shift >= 0; shift -= 8) {
      radix_pass(value, n_slots, shift, mask, prefix, remaining, sh);
      mask |= 255u << shift;
    }
  }
  *tau = prefix;
  *take_eq = remaining;
}

__device__ __forceinline__ void block_minmax(uint32_t lo, uint32_t hi, TopkShared &sh) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (threadIdx.x == 0) { sh.cmin = 0xffffffffu; sh.cmax = 0u; }
  __syncthreads();
  if (lane == 0) { atomicMin(&sh.cmin, lo); atomicMax(&sh.cmax, hi); }
  __syncthreads();
}

// Threshold of the top `need` keys: a 256-key sample, ranked by counting,
// brackets it; one comparison pass counts the keys above the bracket and
// collects those inside it into per-warp segments; an exact radix select on
// the collected keys finishes.  Returns false if the bracket missed or a
// segment overflowed (the caller then selects on all keys).
template <bool kShared>
__device__ __forceinline__ bool bracket_select(const uint32_t *keys, int nc, uint32_t need, TopkShared &sh, uint32_t *cand,
                               uint32_t *tau, uint32_t *take_eq) {
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = kTopkSample;
  if (threadIdx.x < M) sh.sample[threadIdx.x] = key_at<kShared>(keys, (int)(((int64_t)threadIdx.x * nc) / M));
  const double q = (double)need * M / (double)nc;
  const double delta = 4.0 * sqrt(q + 1.0) + 8.0;
  const int r_hi = (int)floor(q - delta);   // 1-based ranks of the bracket ends
  const int r_lo = (int)ceil(q + delta);
  if (threadIdx.x == 0) {
    sh.t_hi = 0xffffffffu;
    sh.t_lo = 0u;
  }
  __syncthreads();
  if (threadIdx.x < M) {
    // rank (0 = largest) by counting; equal keys ordered by sample index
    const uint32_t v = sh.sample[threadIdx.x];
    int rank = 0;
#pragma unroll 8
    for (int j = 0; j < M; ++j) {
      const uint32_t u = sh.sample[j];
      rank += (u > v) || (u == v && j < (int)threadIdx.x);
    }
    if (r_hi >= 1 && rank == r_hi - 1) sh.t_hi = v;
    if (r_lo <= M && rank == r_lo - 1) sh.t_lo = v;
  }
  __syncthreads();
  const uint32_t t_hi = sh.t_hi, t_lo = sh.t_lo;
  // Count keys strictly above t_hi and collect keys in [t_lo, t_hi].
  uint32_t above = 0, seg = 0, cmin = 0xffffffffu, cmax = 0u;
  uint32_t *mine = cand + wid * kTopkSeg;
  for (int i0 = 0; i0 < nc; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    const bool valid = i < nc;
    const uint32_t v = valid ? key_at<kShared>(keys, i) : 0u;
    above += (valid && v > t_hi);
    const bool in = valid && v <= t_hi && v >= t_lo;
    const uint32_t ball = __ballot_sync(0xffffffffu, in);
    if (in) {
      const uint32_t slot = seg + __popc(ball & ((1u << lane) - 1u));
      if (slot < kTopkSeg) mine[slot] = v;
      cmin = min(cmin, v);
      cmax = max(cmax, v);
    }
    seg += __popc(ball);
  }
  above = warp_sum_u32(above);
  if (lane == 0) {
    sh.seg_count[wid] = seg;
    sh.seg_above[wid] = above;
  }
  block_minmax(cmin, cmax, sh);   // includes a __syncthreads
  uint32_t n_above = 0, n_cand = 0;
  bool overflow = false;
  for (int w = 0; w < kTopkWarps; ++w) {
    n_above += sh.seg_above[w];
    n_cand += sh.seg_count[w];
    overflow |= sh.seg_count[w] > (uint32_t)kTopkSeg;
  }
  if (overflow || !(n_above < need && need <= n_above + n_cand)) return false;
  auto value = [&](int i, bool &ok) -> uint32_t {
    const int w = i / kTopkSeg, e = i - w * kTopkSeg;
    ok = e < (int)sh.seg_count[w];
    return ok ? cand[i] : 0u;
  };
  radix_select(value, kTopkCand, need - n_above, sh.cmin, sh.cmax, sh, tau, take_eq);
  return true;
}

// Stable compaction in index order: every key > tau and the first take_eq
// keys == tau, written as absolute positions.
template <bool kShared>
__device__ __forceinline__ void compact_selected(const uint32_t *keys, int nc, uint32_t tau, uint32_t take_eq, int32_t n_sink,
                                 int32_t *out, int k, TopkShared &sh) {
  const int chunk = (nc + (int)blockDim.x - 1) / (int)blockDim.x;
  const int i0 = min(nc, (int)threadIdx.x * chunk);
  const int i1 = min(nc, i0 + chunk);
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at<kShared>(keys, i);
    n_gt += key > tau;
    n_eq += key == tau;
  }
  const uint32_t eq_before = block_excl_scan(n_eq, sh.warp_tot, &sh.total);
  const uint32_t eq_take = (eq_before >= take_eq) ? 0u : min(n_eq, take_eq - eq_before);
  const uint32_t out_before = block_excl_scan(n_gt + eq_take, sh.warp_tot, &sh.total);
  uint32_t pos = out_before, eq_seen = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at<kShared>(keys, i);
    bool take = key > tau;
    if (key == tau) { take = eq_seen < eq_take; ++eq_seen; }
    if (take && pos < (uint32_t)k) out[pos++] = (int32_t)(n_sink + i);
  }
}

template <bool kShared>
__device__ __forceinline__ void select_top(const uint32_t *keys, int nc, uint32_t need, int32_t n_sink, int32_t *out, int k,
                           TopkShared &sh, uint32_t *cand) {
  uint32_t tau = 0, take_eq = 0;
  if (nc <= 4 * kTopkSample || !bracket_select<kShared>(keys, nc, need, sh, cand, &tau, &take_eq)) {
    auto value = [&](int i, bool &ok) -> uint32_t {
      ok = true;
      return key_at<kShared>(keys, i);
    };
    radix_select(value, nc, need, 0u, 0xffffffffu, sh, &tau, &take_eq);
  }
  compact_selected<kShared>(keys, nc, tau, take_eq, n_sink, out, k, sh);
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(Shape s, const int32_t *__restrict__ lengths, const float *__restrict__ keys_all,
            int32_t *__restrict__ idx, uint32_t *__restrict__ status) {
  extern __shared__ __align__(16) uint32_t topk_dyn[];
  __shared__ TopkShared sh;
  pdl_wait();      // scores come from the preceding kernel
  pdl_trigger();
  const int b = blockIdx.x;
  const int64_t Lraw = lengths[b];
  if (threadIdx.x == 0 && (Lraw < 0 || Lraw > s.cache_rows)) set_status(status, kDevStatusCheck);
  const int64_t L = valid_length(Lraw, s.cache_rows);
  const int64_t nc = n_candidates(L, s.local_window);
  const int k = s.top_k;
  int32_t *out = idx + (int64_t)b * k;
  const uint32_t *gkeys = reinterpret_cast<const uint32_t *>(keys_all + (int64_t)b * s.cache_rows);
  const int64_t need = smin<int64_t>(k, nc);
  for (int e = threadIdx.x; e < k; e += blockDim.x)
    if (e >= need) out[e] = -1;
  if (need == 0) return;
  if (need == nc) {
    for (int64_t i = threadIdx.x; i < nc; i += blockDim.x) out[i] = (int32_t)(s.n_sink + i);
    return;
  }
  const int n_stage = kpad((int)smin<int64_t>(s.cache_rows, kTopkSmemKeys)) + 1;
  uint32_t *keys_s = topk_dyn;
  uint32_t *cand = topk_dyn + n_stage;
  if (nc <= kTopkSmemKeys) {
    // Row b starts at b * cache_rows floats, which need not be 16-byte
    // aligned: copy the head up to the first aligned key one by one, the
    // aligned middle with 16-byte loads, and the tail one by one.
    const int64_t head = smin<int64_t>(nc, (int64_t)((16u - (reinterpret_cast<uintptr_t>(gkeys) & 15u)) & 15u) / 4);
    const int64_t n4 = (nc - head) / 4;
    const uint4 *src4 = reinterpret_cast<const uint4 *>(gkeys + head);
    for (int i = threadIdx.x; i < (int)head; i += blockDim.x) keys_s[kpad(i)] = __ldcg(gkeys + i);
    for (int64_t i0 = 0; i0 < n4; i0 += 4 * kTopkThreads) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = i0 + u * kTopkThreads + threadIdx.x;
        if (i < n4) v[u] = __ldcg(src4 + i);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = i0 + u * kTopkThreads + threadIdx.x;
        if (i < n4) {
          const int j = (int)(head + 4 * i);
          keys_s[kpad(j)] = v[u].x;
          keys_s[kpad(j + 1)] = v[u].y;
          keys_s[kpad(j + 2)] = v[u].z;
          keys_s[kpad(j + 3)] = v[u].w;
        }
      }
    }
    for (int i = (int)(head + 4 * n4) + threadIdx.x; i < (int)nc; i += blockDim.x) keys_s[kpad(i)] = __ldcg(gkeys + i);
    __syncthreads();
    select_top<true>(keys_s, (int)nc, (uint32_t)need, s.n_sink, out, k, sh, cand);
  } else {
    select_top<false>(gkeys, (int)nc, (uint32_t)need, s.n_sink, out, k, sh, cand);
  }
}

// ---------------------------------------------------------------------------
// Cluster variant: the kTopkCl CTAs of a cluster split one problem's
// candidates into contiguous shares held in shared memory.  The threshold
// key tau (of the IEEE bit patterns, which order like the scores) is found
// by narrowing a key range [lo, hi] that holds it:
//   * level 0 bins the keys around the mean score (score_bin: steps of 1/256
//     of a binade); its histogram comes from the scoring kernel, or from
//     every rank's histogram of its keys exchanged through distributed shared
//     memory; every rank takes the same decision: the bin holding the
//     remaining-th largest key, and so its key range;
//   * if that range holds at most kTopkGather keys, every rank publishes its
//     keys in it (with their positions, in position order) and its count of
//     keys above it; after one cluster barrier every rank reads them all,
//     finds tau among the gathered keys by a radix select and knows every
//     rank's counts of keys > tau and == tau;
//   * a range taken whole needs only the ranks' counts; a single key value
//     fixes tau; a fuller range is split again into at most 4096 bins.
// Usually that is one exchange.  No keys move except those in the range.
// A stable compaction in index order then writes the rank's keys > tau and
// its share of the keys == tau (lower positions first).
constexpr int kTopkCl = 8;                       // CTAs per problem
constexpr int kTopkClThreads = 512;
constexpr int kTopkClKeys = 16384;               // keys per CTA (64 KB)
constexpr int kTopkLvlBins = 4096;               // bins of levels 0 and 1
constexpr int kTopkGather = 8192;                // keys of the threshold bin gathered into every rank at most
static_assert(kTopkLvlBins == kExpBins, "level 0 uses the scoring histogram's bins");

struct __align__(16) TopkClShared {
  uint32_t hist[kTopkLvlBins];              // summed histogram of the current level
  union {
    // this rank's histogram of a level (two in flight), read by every rank
    uint32_t pub_hist[2][kTopkLvlBins];
    // every rank's keys of the threshold bin, rank order: written only after
    // the exchange barrier, which every rank passes after its last read of
    // the histograms
    uint2 gath[kTopkGather];
  };
  uint2 pub_cand[kTopkGather];              // this rank's keys of the threshold bin (key, position), position order
  uint32_t pub_hdr[4];                      // this rank's count of keys above the bin, of keys in it
  uint32_t g_gt[kTopkCl], g_n[kTopkCl], g_off[kTopkCl + 1];
  uint32_t gt_acc[kTopkCl], eq_acc[kTopkCl];  // every rank's keys > tau / == tau
  uint32_t sel_hist[256];
  uint32_t warp_tot[32];
  uint32_t total, digit, above, mode, out_before, eq_before;
};
__host__ inline size_t topk_cl_smem_bytes() {
  return sizeof(TopkClShared) + sizeof(uint32_t) * ((size_t)kpad(kTopkClKeys) + 1);
}

// Shift and number of bins of digit level l.
__device__ __forceinline__ int cl_shift(int l) { return l == 0 ? 19 : (l == 1 ? 7 : 0); }
__device__ __forceinline__ int cl_bins(int l) { return l < 2 ? kTopkLvlBins : 128; }

// The bin (from the top) of `hist` holding the remaining-th largest key, and
// how many keys lie in higher bins: sh.digit, sh.above.  Thread t owns bins
// nbins-1-8t .. nbins-8-8t; a block scan orders the threads' counts.
__device__ __forceinline__ void cl_pick_bin(TopkClShared &sh, const uint32_t *hist, int nbins, uint32_t remaining) {
  uint32_t cnt[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int b = nbins - 1 - (8 * (int)threadIdx.x + j);
    cnt[j] = b >= 0 ? hist[b] : 0u;
    sum += cnt[j];
  }
  uint32_t run = block_excl_scan(sum, sh.warp_tot, &sh.total);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (run < remaining && run + cnt[j] >= remaining) {
      sh.digit = (uint32_t)(nbins - 1 - (8 * (int)threadIdx.x + j));
      sh.above = run;
    }
    run += cnt[j];
  }
  __syncthreads();
}

// Warp 0: the digit (from the top) of a 256-bin histogram holding the
// remaining-th largest key, and the count in higher bins.
__device__ __forceinline__ void cl_pick_digit256(TopkClShared &sh, const uint32_t *hist, uint32_t remaining) {
  const int lane = threadIdx.x & 31;
  uint32_t cnt[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) { cnt[j] = hist[255 - (lane * 8 + j)]; sum += cnt[j]; }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t run = incl - sum;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (run < remaining && run + cnt[j] >= remaining) {
      sh.digit = 255u - (uint32_t)(lane * 8 + j);
      sh.above = run;
    }
    run += cnt[j];
  }
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint2 ld_cluster_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared::cluster.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr) : "memory");
  return v;
}

__global__ void __cluster_dims__(kTopkCl, 1, 1) __launch_bounds__(kTopkClThreads, 1)
topk_cluster_kernel(Shape s, const int32_t *__restrict__ lengths, const float *__restrict__ keys_all,
                    const uint32_t *__restrict__ ehist, int32_t *__restrict__ idx, uint32_t *__restrict__ status) {
  extern __shared__ __align__(16) unsigned char tcl_dyn[];
  TopkClShared &sh = *reinterpret_cast<TopkClShared *>(tcl_dyn);
  uint32_t *keys_s = reinterpret_cast<uint32_t *>(tcl_dyn + sizeof(TopkClShared));   // this rank's keys (padded)
  pdl_wait();      // scores come from the preceding kernel
  pdl_trigger();
  const uint32_t rank = cluster_ctarank();
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t Lraw = lengths[b];
  if (rank == 0 && threadIdx.x == 0 && (Lraw < 0 || Lraw > s.cache_rows)) set_status(status, kDevStatusCheck);
  const int64_t L = valid_length(Lraw, s.cache_rows);
  const int nc = (int)n_candidates(L, s.local_window);
  const int k = s.top_k;
  int32_t *out = idx + (int64_t)b * k;
  const uint32_t *gkeys = reinterpret_cast<const uint32_t *>(keys_all + (int64_t)b * s.cache_rows);
  const int need = min(k, nc);
  // Trivial cases: every rank takes the same branch (uniform), no cluster barrier used.
  if (need == 0 || need == nc) {
    for (int e = (int)rank * blockDim.x + threadIdx.x; e < k; e += kTopkCl * blockDim.x)
      out[e] = (e < nc) ? (int32_t)(s.n_sink + e) : -1;
    return;
  }
  for (int e = need + (int)rank * blockDim.x + threadIdx.x; e < k; e += kTopkCl * blockDim.x) out[e] = -1;
  const int chunk = (nc + kTopkCl - 1) / kTopkCl;
  const int i_begin = min(nc, (int)rank * chunk), i_end = min(nc, i_begin + chunk);
  const int my_n = i_end - i_begin;
  // Level 0 from the scoring kernel's histogram: 16-byte loads issued before
  // the keys', stored after them, so the two reads overlap.
  constexpr int kHistV = kTopkLvlBins / 4 / kTopkClThreads;   // 16-byte words per thread
  static_assert(kTopkLvlBins % (4 * kTopkClThreads) == 0, "histogram words per thread");
  uint4 hv[kHistV];
  if (ehist != nullptr) {
    const uint4 *src = reinterpret_cast<const uint4 *>(ehist + (int64_t)b * kExpBins);
#pragma unroll
    for (int u = 0; u < kHistV; ++u) hv[u] = __ldcg(src + u * kTopkClThreads + threadIdx.x);
  }
  // Stage the share with 16-byte loads, all in flight at once.  The share
  // starts at key i_begin of a row that starts at b * cache_rows floats, so
  // it need not be 16-byte aligned: the head up to the first aligned key and
  // the tail go one by one.
  {
    const uint32_t *src = gkeys + i_begin;
    const int head = min(my_n, (int)(((16u - (reinterpret_cast<uintptr_t>(src) & 15u)) & 15u) / 4));
    const int n4 = (my_n - head) / 4;
    const uint4 *src4 = reinterpret_cast<const uint4 *>(src + head);
    for (int i = threadIdx.x; i < head; i += blockDim.x) keys_s[kpad(i)] = __ldcg(src + i);
    for (int i0 = 0; i0 < n4; i0 += 4 * (int)blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
        if (i < n4) v[u] = __ldcg(src4 + i);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
        if (i < n4) {
          const int j = head + 4 * i;
          keys_s[kpad(j)] = v[u].x;
          keys_s[kpad(j + 1)] = v[u].y;
          keys_s[kpad(j + 2)] = v[u].z;
          keys_s[kpad(j + 3)] = v[u].w;
        }
      }
    }
    for (int i = head + 4 * n4 + (int)threadIdx.x; i < my_n; i += blockDim.x) keys_s[kpad(i)] = __ldcg(src + i);
  }
  if (ehist != nullptr) {
#pragma unroll
    for (int u = 0; u < kHistV; ++u) reinterpret_cast<uint4 *>(sh.hist)[u * kTopkClThreads + threadIdx.x] = hv[u];
  }
  __syncthreads();

  // Per-thread contiguous chunk of the rank's keys (the compactions walk it).
  const int per = (my_n + (int)blockDim.x - 1) / (int)blockDim.x;
  const int j0 = min(my_n, (int)threadIdx.x * per), j1 = min(my_n, j0 + per);

  const uint32_t center = score_center(s.n_rows, L);
  uint32_t lo = 0u, hi = 0x7fffffffu, remaining = (uint32_t)need, in_bin = 0u;
  uint32_t tau = 0u, take_eq = 0u;
  int mode = 0;              // 1: range taken whole; 2: a single key value; 3: range gathered
  for (int level = 0; level < 6; ++level) {
    // Bins of this level: score_bin at level 0, else (key - lo) >> sh over [lo, hi].
    const uint32_t w = hi - lo;
    const int bsh = level == 0 ? 0 : ((w >> 12) == 0u ? 0 : 32 - __clz(w >> 12));
    const int nbins = level == 0 ? kTopkLvlBins : (int)(w >> bsh) + 1;
    if (level > 0 || ehist == nullptr) {
      // This rank's histogram of its keys in [lo, hi], summed over the ranks
      // through distributed shared memory.
      uint32_t *ph = sh.pub_hist[level & 1];
      for (int i = threadIdx.x; i < kTopkLvlBins; i += blockDim.x) ph[i] = 0u;
      __syncthreads();
      for (int i = threadIdx.x; i < my_n; i += blockDim.x) {
        const uint32_t v = keys_s[kpad(i)];
        if (level == 0) atomicAdd(&ph[score_bin(v, center)], 1u);
        else if (v >= lo && v <= hi) atomicAdd(&ph[(v - lo) >> bsh], 1u);
      }
      cluster_sync();
      for (int i = 4 * (int)threadIdx.x; i < nbins; i += 4 * (int)blockDim.x) {
        uint4 acc = make_uint4(0u, 0u, 0u, 0u);
        for (int rr = 0; rr < kTopkCl; ++rr) {
          const uint4 v = ld_cluster_v4(cluster_map(&ph[i], (uint32_t)rr));
          acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        *reinterpret_cast<uint4 *>(&sh.hist[i]) = acc;
      }
      __syncthreads();
    }
    cl_pick_bin(sh, sh.hist, nbins, remaining);
    const uint32_t d = sh.digit;
    in_bin = sh.hist[d];
    remaining -= sh.above;
    if (level == 0) {
      score_bin_range((int)d, center, lo, hi);
    } else {
      const uint32_t nlo = lo + (d << bsh);
      const uint32_t top = nlo + ((1u << bsh) - 1u);
      hi = top < hi ? top : hi;
      lo = nlo;
    }
    __syncthreads();
    if (in_bin == remaining && lo > 0u) {
      mode = 1;                    // every key >= lo is taken
      tau = lo - 1u;
      take_eq = 0u;
      break;
    }
    if (lo == hi) {
      mode = 2;                    // the range is a single key value
      tau = lo;
      take_eq = remaining;
      break;
    }
    if (in_bin <= (uint32_t)kTopkGather) {
      mode = 3;
      break;
    }
  }

  if (mode == 3) {
    // Publish this rank's keys of the bin (stable, in position order) and
    // its count of keys above the bin; gather every rank's.
    uint32_t n_in = 0, n_above = 0;
    for (int i = j0; i < j1; ++i) {
      const uint32_t v = keys_s[kpad(i)];
      n_in += v >= lo && v <= hi;
      n_above += v > hi;
    }
    const uint32_t before = block_excl_scan(n_in, sh.warp_tot, &sh.total);
    uint32_t at = before;
    for (int i = j0; i < j1; ++i) {
      const uint32_t v = keys_s[kpad(i)];
      if (v >= lo && v <= hi) sh.pub_cand[at++] = make_uint2(v, (uint32_t)(i_begin + i));
    }
    n_above = warp_sum_u32(n_above);
    if (threadIdx.x == 0) { sh.pub_hdr[0] = 0u; sh.pub_hdr[1] = sh.total; }
    __syncthreads();
    if (lane == 0 && n_above) atomicAdd(&sh.pub_hdr[0], n_above);
    cluster_sync();
    if (threadIdx.x < kTopkCl) {
      sh.g_gt[threadIdx.x] = ld_cluster_u32(cluster_map(&sh.pub_hdr[0], threadIdx.x));
      sh.g_n[threadIdx.x] = ld_cluster_u32(cluster_map(&sh.pub_hdr[1], threadIdx.x));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t o = 0;
      for (int rr = 0; rr < kTopkCl; ++rr) { sh.g_off[rr] = o; o += sh.g_n[rr]; }
      sh.g_off[kTopkCl] = o;
    }
    __syncthreads();
    const uint32_t n_g = sh.g_off[kTopkCl];   // == in_bin <= kTopkGather
    for (uint32_t e = threadIdx.x; e < n_g; e += blockDim.x) {
      int rr = 0;
      while (rr + 1 < kTopkCl && e >= sh.g_off[rr + 1]) ++rr;
      sh.gath[e] = ld_cluster_v2(cluster_map(&sh.pub_cand[e - sh.g_off[rr]], (uint32_t)rr));
    }
    __syncthreads();
    // tau: the remaining-th largest gathered key, by a radix select on the
    // offsets v = key - lo (at most hi - lo), 8 bits at a time from the top.
    uint32_t pfx = 0u, msk = 0u, rem = remaining;
    for (int top = 31 - __clz(hi - lo); top >= 0;) {
      const int sh8 = top >= 7 ? top - 7 : 0;
      for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.sel_hist[i] = 0u;
      __syncthreads();
      for (uint32_t e = threadIdx.x; e < n_g; e += blockDim.x) {
        const uint32_t v = sh.gath[e].x - lo;
        if ((v & msk) == pfx) atomicAdd(&sh.sel_hist[(v >> sh8) & 255u], 1u);
      }
      __syncthreads();
      if (threadIdx.x < 32) cl_pick_digit256(sh, sh.sel_hist, rem);
      __syncthreads();
      rem -= sh.above;
      pfx |= sh.digit << sh8;
      msk |= 255u << sh8;
      __syncthreads();
      top = sh8 - 1;
    }
    tau = lo + pfx;
    take_eq = rem;
    // Every rank's keys > tau and == tau: those above the bin plus its gathered keys.
    if (threadIdx.x < kTopkCl) { sh.gt_acc[threadIdx.x] = sh.g_gt[threadIdx.x]; sh.eq_acc[threadIdx.x] = 0u; }
    __syncthreads();
    for (uint32_t e = threadIdx.x; e < n_g; e += blockDim.x) {
      int rr = 0;
      while (rr + 1 < kTopkCl && e >= sh.g_off[rr + 1]) ++rr;
      const uint32_t v = sh.gath[e].x;
      if (v > tau) atomicAdd(&sh.gt_acc[rr], 1u);
      else if (v == tau) atomicAdd(&sh.eq_acc[rr], 1u);
    }
  } else {
    // Modes 1 and 2: only every rank's counts of keys > tau and == tau.
    uint32_t n_gt = 0, n_eq = 0;
    for (int i = j0; i < j1; ++i) {
      const uint32_t v = keys_s[kpad(i)];
      n_gt += v > tau;
      n_eq += v == tau;
    }
    n_gt = warp_sum_u32(n_gt);
    n_eq = warp_sum_u32(n_eq);
    if (threadIdx.x == 0) { sh.pub_hdr[2] = 0u; sh.pub_hdr[3] = 0u; }
    __syncthreads();
    if (lane == 0) {
      if (n_gt) atomicAdd(&sh.pub_hdr[2], n_gt);
      if (n_eq) atomicAdd(&sh.pub_hdr[3], n_eq);
    }
    cluster_sync();
    if (threadIdx.x < kTopkCl) {
      sh.gt_acc[threadIdx.x] = ld_cluster_u32(cluster_map(&sh.pub_hdr[2], threadIdx.x));
      sh.eq_acc[threadIdx.x] = ld_cluster_u32(cluster_map(&sh.pub_hdr[3], threadIdx.x));
    }
  }
  // Every read of another rank's shared memory is done; the ranks learn that
  // theirs have been read only here, so no rank leaves before all arrive.
  // The arrive publishes no data, hence relaxed.
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  __syncthreads();
  (void)wid;
  if (threadIdx.x == 0) {
    uint32_t out_before = 0, eq_before = 0;
    for (uint32_t c = 0; c < rank; ++c) {
      const uint32_t eq2 = sh.eq_acc[c];
      const uint32_t take2 = (eq_before >= take_eq) ? 0u : min(eq2, take_eq - eq_before);
      out_before += sh.gt_acc[c] + take2;
      eq_before += eq2;
    }
    sh.out_before = out_before;
    sh.eq_before = eq_before;
  }
  __syncthreads();
  const uint32_t out_before_rank = sh.out_before, eq_before_rank = sh.eq_before;
  // Per-thread contiguous chunks: one scan of (n_gt << 16 | n_eq), which
  // cannot carry between the halves because a rank holds < 65536 keys.
  static_assert(kTopkClKeys < 65536, "packed counts");
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = j0; i < j1; ++i) {
    const uint32_t key = keys_s[kpad(i)];
    n_gt += key > tau;
    n_eq += key == tau;
  }
  const uint32_t packed_before = block_excl_scan((n_gt << 16) | n_eq, sh.warp_tot, &sh.total);
  const uint32_t eq_before_local = packed_before & 0xffffu, gt_before_local = packed_before >> 16;
  // Equal keys still to take when this rank starts, and this thread's share.
  const uint32_t avail = take_eq > eq_before_rank ? take_eq - eq_before_rank : 0u;
  const uint32_t take_before_local = min(avail, eq_before_local);
  const uint32_t eq_take = avail > eq_before_local ? min(n_eq, avail - eq_before_local) : 0u;
  uint32_t pos = out_before_rank + gt_before_local + take_before_local, eq_seen = 0;
  for (int i = j0; i < j1; ++i) {
    const uint32_t key = keys_s[kpad(i)];
    bool take = key > tau;
    if (key == tau) { take = eq_seen < eq_take; ++eq_seen; }
    if (take && pos < (uint32_t)k) out[pos++] = (int32_t)(s.n_sink + i_begin + i);
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace s4r
