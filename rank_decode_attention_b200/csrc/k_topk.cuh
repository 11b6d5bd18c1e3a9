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
constexpr int kTopkBins = 2048;
__host__ inline size_t topk_smem_bytes(int64_t cache_rows) {
  return sizeof(uint32_t) * (size_t)smin<int64_t>(cache_rows, kTopkSmemKeys);
}

// Histogram update aggregated across the lanes of a warp that share a bin
// (scores of one problem share their high bits, so plain atomics serialise).
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t bin, bool active) {
  const uint32_t key = active ? bin : 0xffffffffu;
  const uint32_t peers = __match_any_sync(0xffffffffu, key);
  const int leader = __ffs(peers) - 1;
  if (active && (threadIdx.x & 31) == leader) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(Shape s, const int32_t *__restrict__ lengths, const float *__restrict__ keys_all,
            int32_t *__restrict__ idx, uint32_t *__restrict__ status) {
  extern __shared__ __align__(16) uint32_t topk_keys_s[];
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
    const int64_t n4 = nc / 4;
    const uint4 *src4 = reinterpret_cast<const uint4 *>(gkeys);
    uint4 *dst4 = reinterpret_cast<uint4 *>(topk_keys_s);
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
        if (i < n4) dst4[i] = v[u];
      }
    }
    for (int64_t i = n4 * 4 + threadIdx.x; i < nc; i += blockDim.x) topk_keys_s[i] = __ldcg(gkeys + i);
    __syncthreads();
  }
  const uint32_t *keys = staged ? topk_keys_s : gkeys;
  // Radix select of the need-th largest key: digits of 11, 11 and 10 bits.
  uint32_t prefix = 0, mask = 0;
  uint32_t remaining = (uint32_t)need;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const uint32_t nb = 1u << widths[pass], dmask = nb - 1u;
    for (int e = threadIdx.x; e < (int)nb; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    for (int64_t i0 = 0; i0 < nc; i0 += 4 * (int64_t)blockDim.x) {
      uint32_t kv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // loads first, so up to 4 are in flight
        const int64_t i = i0 + u * (int64_t)blockDim.x + threadIdx.x;
        kv[u] = (i < nc) ? keys[i] : 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = i0 + u * (int64_t)blockDim.x + threadIdx.x;
        const bool act = (i < nc) && ((kv[u] & mask) == prefix);
        hist_add(hist, (kv[u] >> shift) & dmask, act);
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // Warp 0 walks the bins from the top; lane l owns nb/32 consecutive bins.
      const int lane = threadIdx.x;
      const int per = (int)nb / 32;
      uint32_t sum = 0;
      for (int j = 0; j < per; ++j) sum += hist[nb - 1 - (lane * per + j)];
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t run = incl - sum;
      if (run < remaining && incl >= remaining) {
        for (int j = 0; j < per; ++j) {
          const uint32_t bin = nb - 1 - (uint32_t)(lane * per + j);
          const uint32_t c = hist[bin];
          if (run + c >= remaining) {
            sh_digit = bin;
            sh_above = run;
            break;
          }
          run += c;
        }
      }
    }
    __syncthreads();
    remaining -= sh_above;
    prefix |= sh_digit << shift;
    mask |= dmask << shift;
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
    const uint32_t key = keys[i];
    n_gt += key > tau;
    n_eq += key == tau;
  }
  const uint32_t eq_before = block_excl_scan(n_eq, warp_tot, &sh_total);
  const uint32_t eq_take = (eq_before >= take_eq) ? 0u : min(n_eq, take_eq - eq_before);
  const uint32_t out_before = block_excl_scan(n_gt + eq_take, warp_tot, &sh_total);
  uint32_t pos = out_before, eq_seen = 0;
  for (int64_t i = i0; i < i1; ++i) {
    const uint32_t key = keys[i];
    bool take = key > tau;
    if (key == tau) { take = eq_seen < eq_take; ++eq_seen; }
    if (take && pos < (uint32_t)k) out[pos++] = (int32_t)(s.n_sink + i);
  }
}

}  // namespace s4r
