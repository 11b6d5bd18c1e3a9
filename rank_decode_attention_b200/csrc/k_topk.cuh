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

namespace s4r {

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ int64_t valid_length(int64_t L, int64_t cap) {
  return (L >= 0 && L <= cap) ? L : 0;
}

// Max-pool of candidate scores, stride 1, same padding, odd kernel.
__global__ void pool_kernel(Shape s, const int32_t *__restrict__ lengths,
                            const float *__restrict__ scores, float *__restrict__ pooled) {
  const int b = blockIdx.y;
  const int64_t L = valid_length(lengths[b], s.cache_rows);
  const int64_t nc = n_candidates(L, s.local_window);
  const int half = s.pool_kernel / 2;
  const float *sb = scores + (int64_t)b * s.cache_rows;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nc;
       i += (int64_t)gridDim.x * blockDim.x) {
    float m = sb[i];
    for (int64_t j = smax<int64_t>(0, i - half); j <= smin<int64_t>(nc - 1, i + half); ++j)
      m = fmaxf(m, sb[j]);
    pooled[(int64_t)b * s.cache_rows + i] = m;
  }
}

// Inclusive block scan of one value per thread (kTopkThreads threads).
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
    uint32_t t = warp_tot[lane];
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
__host__ __device__ __forceinline__ int64_t kpad(int64_t i) { return i + (i >> 5); }
constexpr int kTopkBins = 256;         // 8-bit digits
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSample = 1024;      // sampled keys that bracket the threshold
constexpr int kTopkCand = 8192;        // capacity of the in-bracket candidate list
__host__ inline size_t topk_smem_bytes(int64_t cache_rows) {
  return sizeof(uint32_t) * ((size_t)kpad(smin<int64_t>(cache_rows, kTopkSmemKeys)) + 1 + kTopkCand);
}

struct TopkShared {
  uint32_t whist[kTopkWarps][kTopkBins];
  uint32_t hist[kTopkBins];
  uint32_t sample[kTopkSample];
  uint32_t warp_tot[32];
  uint32_t total, digit, above, n_cand, n_above;
};

// Exact radix select over a short shared-memory array: the value tau of the
// need-th largest element (1 <= need <= n) and how many elements equal to tau
// belong to the top `need`.  Per-warp histograms; contention stays small
// because n is small.
__device__ void radix_select_small(const uint32_t *vals, int n, uint32_t need, TopkShared &sh, uint32_t *tau_out,
                                   uint32_t *take_eq_out) {
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0, remaining = need;
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int j = 0; j < kTopkBins / 32; ++j) sh.whist[wid][lane + 32 * j] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t v = vals[i];
      if ((v & mask) == prefix) atomicAdd(&sh.whist[wid][(v >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < kTopkBins) {
      uint32_t c = 0;
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
    mask |= 255u << shift;
    __syncthreads();
  }
  *tau_out = prefix;
  *take_eq_out = remaining;
}

template <bool kShared>
__device__ __forceinline__ uint32_t key_at(const uint32_t *keys, int64_t i) {
  return kShared ? keys[kpad(i)] : __ldcg(keys + i);
}

// Threshold of the top `need` keys: a sorted-free sample brackets it, one
// comparison pass counts the keys above the bracket and collects those inside
// it, and an exact radix select on the collected keys finishes.  Returns false
// if the bracket missed or overflowed the candidate list (the caller then
// selects on all keys).
template <bool kShared>
__device__ bool bracket_select(const uint32_t *keys, int64_t nc, uint32_t need, TopkShared &sh, uint32_t *cand,
                               uint32_t *tau, uint32_t *take_eq) {
  const int lane = threadIdx.x & 31;
  // Sample and two of its order statistics around the expected rank.
  const int M = kTopkSample;
  for (int i = threadIdx.x; i < M; i += blockDim.x) sh.sample[i] = key_at<kShared>(keys, (int64_t)i * nc / M);
  __syncthreads();
  const double q = (double)need * M / (double)nc;
  const double delta = 4.0 * sqrt(q + 1.0) + 8.0;
  const int r_hi = (int)fmax(1.0, floor(q - delta));       // rank (1-based) of the upper bracket end
  const int r_lo = (int)fmin((double)M, ceil(q + delta));   // rank of the lower bracket end
  uint32_t t_hi = 0xffffffffu, t_lo = 0u, dummy;
  if (q - delta >= 1.0) radix_select_small(sh.sample, M, (uint32_t)r_hi, sh, &t_hi, &dummy);
  if (q + delta <= (double)M) radix_select_small(sh.sample, M, (uint32_t)r_lo, sh, &t_lo, &dummy);
  // Count keys strictly above t_hi and collect keys in [t_lo, t_hi].
  if (threadIdx.x == 0) { sh.n_cand = 0; sh.n_above = 0; }
  __syncthreads();
  uint32_t above = 0;
  for (int64_t i0 = 0; i0 < nc; i0 += blockDim.x) {
    const int64_t i = i0 + threadIdx.x;
    const uint32_t v = (i < nc) ? key_at<kShared>(keys, i) : 0u;
    const bool valid = i < nc;
    above += (valid && v > t_hi);
    const bool in = valid && v <= t_hi && v >= t_lo;
    const uint32_t ball = __ballot_sync(0xffffffffu, in);
    uint32_t base = 0;
    if (lane == 0 && ball) base = atomicAdd(&sh.n_cand, (uint32_t)__popc(ball));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (in) {
      const uint32_t slot = base + __popc(ball & ((1u << lane) - 1u));
      if (slot < kTopkCand) cand[slot] = v;
    }
  }
  above = warp_sum_u32(above);
  if (lane == 0 && above) atomicAdd(&sh.n_above, above);
  __syncthreads();
  const uint32_t n_above = sh.n_above, n_cand = sh.n_cand;
  if (!(n_above < need && need <= n_above + n_cand) || n_cand > (uint32_t)kTopkCand) return false;
  radix_select_small(cand, (int)n_cand, need - n_above, sh, tau, take_eq);
  return true;
}

// Exact radix select over all keys (fallback).
template <bool kShared>
__device__ void radix_select_all(const uint32_t *keys, int64_t nc, uint32_t need, TopkShared &sh, uint32_t *tau,
                                 uint32_t *take_eq) {
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0, remaining = need;
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int j = 0; j < kTopkBins / 32; ++j) sh.whist[wid][lane + 32 * j] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < nc; i += blockDim.x) {
      const uint32_t v = key_at<kShared>(keys, i);
      if ((v & mask) == prefix) atomicAdd(&sh.whist[wid][(v >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < kTopkBins) {
      uint32_t c = 0;
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
    mask |= 255u << shift;
    __syncthreads();
  }
  *tau = prefix;
  *take_eq = remaining;
}

// Stable compaction in index order: every key > tau and the first take_eq
// keys == tau, written as absolute positions.
template <bool kShared>
__device__ void compact_selected(const uint32_t *keys, int64_t nc, uint32_t tau, uint32_t take_eq, int32_t n_sink,
                                 int32_t *out, int k, TopkShared &sh) {
  const int64_t chunk = ceil_div(nc, blockDim.x);
  const int64_t i0 = smin<int64_t>(nc, (int64_t)threadIdx.x * chunk);
  const int64_t i1 = smin<int64_t>(nc, i0 + chunk);
  uint32_t n_gt = 0, n_eq = 0;
  for (int64_t i = i0; i < i1; ++i) {
    const uint32_t key = key_at<kShared>(keys, i);
    n_gt += key > tau;
    n_eq += key == tau;
  }
  const uint32_t eq_before = block_excl_scan(n_eq, sh.warp_tot, &sh.total);
  const uint32_t eq_take = (eq_before >= take_eq) ? 0u : min(n_eq, take_eq - eq_before);
  const uint32_t out_before = block_excl_scan(n_gt + eq_take, sh.warp_tot, &sh.total);
  uint32_t pos = out_before, eq_seen = 0;
  for (int64_t i = i0; i < i1; ++i) {
    const uint32_t key = key_at<kShared>(keys, i);
    bool take = key > tau;
    if (key == tau) { take = eq_seen < eq_take; ++eq_seen; }
    if (take && pos < (uint32_t)k) out[pos++] = (int32_t)(n_sink + i);
  }
}

template <bool kShared>
__device__ void select_top(const uint32_t *keys, int64_t nc, uint32_t need, int32_t n_sink, int32_t *out, int k,
                           TopkShared &sh, uint32_t *cand) {
  uint32_t tau = 0, take_eq = 0;
  if (nc <= 2 * kTopkSample || !bracket_select<kShared>(keys, nc, need, sh, cand, &tau, &take_eq))
    radix_select_all<kShared>(keys, nc, need, sh, &tau, &take_eq);
  compact_selected<kShared>(keys, nc, tau, take_eq, n_sink, out, k, sh);
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(Shape s, const int32_t *__restrict__ lengths, const float *__restrict__ keys_all,
            int32_t *__restrict__ idx, uint32_t *__restrict__ status) {
  extern __shared__ __align__(16) uint32_t topk_dyn[];
  __shared__ TopkShared sh;
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
  const int64_t n_stage = kpad(smin<int64_t>(s.cache_rows, kTopkSmemKeys)) + 1;
  uint32_t *keys_s = topk_dyn;
  uint32_t *cand = topk_dyn + n_stage;
  if (nc <= kTopkSmemKeys) {
    // Row b starts at b * cache_rows floats, which need not be 16-byte
    // aligned: copy the head up to the first aligned key one by one, the
    // aligned middle with 16-byte loads, and the tail one by one.
    const int64_t head = smin<int64_t>(nc, (int64_t)((16u - (reinterpret_cast<uintptr_t>(gkeys) & 15u)) & 15u) / 4);
    const int64_t n4 = (nc - head) / 4;
    const uint4 *src4 = reinterpret_cast<const uint4 *>(gkeys + head);
    for (int64_t i = threadIdx.x; i < head; i += blockDim.x) keys_s[kpad(i)] = __ldcg(gkeys + i);
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
          const int64_t j = head + 4 * i;
          keys_s[kpad(j)] = v[u].x;
          keys_s[kpad(j + 1)] = v[u].y;
          keys_s[kpad(j + 2)] = v[u].z;
          keys_s[kpad(j + 3)] = v[u].w;
        }
      }
    }
    for (int64_t i = head + 4 * n4 + threadIdx.x; i < nc; i += blockDim.x) keys_s[kpad(i)] = __ldcg(gkeys + i);
    __syncthreads();
    select_top<true>(keys_s, nc, (uint32_t)need, s.n_sink, out, k, sh, cand);
  } else {
    select_top<false>(gkeys, nc, (uint32_t)need, s.n_sink, out, k, sh, cand);
  }
}

}  // namespace s4r
