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

constexpr int kTopkSmemKeys = 40960;  // keys staged in shared memory (160 KB) when they fit
constexpr int kTopkBins = 256;     // 8-bit digits, 4 passes
constexpr int kTopkWarps = kTopkThreads / 32;
__host__ inline size_t topk_smem_bytes(int64_t cache_rows) {
  return sizeof(uint32_t) * (size_t)smin<int64_t>(cache_rows, kTopkSmemKeys);
}

// One histogram pass over the keys into the calling warp's private
// histogram.  Scores of one problem share their high bits, so atomics on a
// shared histogram serialise; instead each warp loops over the distinct
// digits present among its 32 lanes (one ballot per digit, usually one to
// three in the high passes, and few keys are still active in the low
// passes) and lane 0 alone updates the warp's histogram.
template <bool kShared>
__device__ __forceinline__ void hist_pass(const uint32_t *keys, int64_t nc, uint32_t mask, uint32_t prefix,
                                          int shift, uint32_t *whist) {
  const int lane = threadIdx.x & 31;
  for (int64_t i0 = 0; i0 < nc; i0 += 4 * (int64_t)blockDim.x) {
    uint32_t kv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * (int64_t)blockDim.x + threadIdx.x;
      kv[u] = (i < nc) ? (kShared ? keys[i] : __ldcg(keys + i)) : 0u;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * (int64_t)blockDim.x + threadIdx.x;
      const bool act = (i < nc) && ((kv[u] & mask) == prefix);
      const uint32_t d = (kv[u] >> shift) & 255u;
      uint32_t pending = __ballot_sync(0xffffffffu, act);
      while (pending) {
        const uint32_t dd = __shfl_sync(0xffffffffu, d, __ffs(pending) - 1);
        const uint32_t same = __ballot_sync(0xffffffffu, d == dd) & pending;
        if (lane == 0) whist[dd] += (uint32_t)__popc(same);
        pending &= ~same;
      }
    }
  }
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(Shape s, const int32_t *__restrict__ lengths, const float *__restrict__ keys_all,
            int32_t *__restrict__ idx, uint32_t *__restrict__ status) {
  extern __shared__ __align__(16) uint32_t topk_keys_s[];
  __shared__ uint32_t whist[kTopkWarps][kTopkBins];
  __shared__ uint32_t hist[kTopkBins];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t sh_total, sh_digit, sh_above;
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
  // Stage the keys in shared memory when they fit (16-byte loads, all in flight).
  const bool staged = nc <= kTopkSmemKeys;
  if (staged) {
    // Row b starts at b * cache_rows floats, which need not be 16-byte
    // aligned: copy the head up to the first aligned key one by one, the
    // aligned middle with 16-byte loads, and the tail one by one.
    const int64_t head = smin<int64_t>(nc, (int64_t)((16u - (reinterpret_cast<uintptr_t>(gkeys) & 15u)) & 15u) / 4);
    const int64_t n4 = (nc - head) / 4;
    const uint4 *src4 = reinterpret_cast<const uint4 *>(gkeys + head);
    for (int64_t i = threadIdx.x; i < head; i += blockDim.x) topk_keys_s[i] = __ldcg(gkeys + i);
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
          uint32_t *d = topk_keys_s + head + 4 * i;   // shared copy may be unaligned too: scalar stores
          d[0] = v[u].x; d[1] = v[u].y; d[2] = v[u].z; d[3] = v[u].w;
        }
      }
    }
    for (int64_t i = head + 4 * n4 + threadIdx.x; i < nc; i += blockDim.x) topk_keys_s[i] = __ldcg(gkeys + i);
    __syncthreads();
  }
  // Radix select of the need-th largest key, 8-bit digits from the top.
  uint32_t prefix = 0, mask = 0;
  uint32_t remaining = (uint32_t)need;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int j = 0; j < kTopkBins / 32; ++j) whist[wid][lane + 32 * j] = 0;
    __syncwarp();
    if (staged)
      hist_pass<true>(topk_keys_s, nc, mask, prefix, shift, whist[wid]);
    else
      hist_pass<false>(gkeys, nc, mask, prefix, shift, whist[wid]);
    __syncthreads();
    if (threadIdx.x < kTopkBins) {
      uint32_t c = 0;
      for (int w = 0; w < kTopkWarps; ++w) c += whist[w][threadIdx.x];
      hist[threadIdx.x] = c;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // Warp 0 walks the digits from the top, 8 per lane.
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
          sh_digit = 255u - (uint32_t)(lane * 8 + j);
          sh_above = run;
        }
        run += cnt[j];
      }
    }
    __syncthreads();
    remaining -= sh_above;
    prefix |= sh_digit << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const uint32_t take_eq = remaining;  // >= 1 keys equal to tau, lowest index first
  // Stable compaction over contiguous per-thread chunks.
  const int64_t chunk = ceil_div(nc, blockDim.x);
  const int64_t i0 = smin<int64_t>(nc, (int64_t)threadIdx.x * chunk);
  const int64_t i1 = smin<int64_t>(nc, i0 + chunk);
  uint32_t n_gt = 0, n_eq = 0;
  for (int64_t i = i0; i < i1; ++i) {
    const uint32_t key = staged ? topk_keys_s[i] : __ldcg(gkeys + i);
    n_gt += key > tau;
    n_eq += key == tau;
  }
  const uint32_t eq_before = block_excl_scan(n_eq, warp_tot, &sh_total);
  const uint32_t eq_take = (eq_before >= take_eq) ? 0u : min(n_eq, take_eq - eq_before);
  const uint32_t out_before = block_excl_scan(n_gt + eq_take, warp_tot, &sh_total);
  uint32_t pos = out_before, eq_seen = 0;
  for (int64_t i = i0; i < i1; ++i) {
    const uint32_t key = staged ? topk_keys_s[i] : __ldcg(gkeys + i);
    bool take = key > tau;
    if (key == tau) { take = eq_seen < eq_take; ++eq_seen; }
    if (take && pos < (uint32_t)k) out[pos++] = (int32_t)(s.n_sink + i);
  }
}

}  // namespace s4r
