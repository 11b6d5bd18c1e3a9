// common.cuh -- shared device helpers for libs4r (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "s4r.h"

namespace s4r {

// Sticky device status bits (workspace word 0).
constexpr uint32_t kDevStatusCheck = 1u;    // a device-side check failed -> S4R_ERR_DEVICE
constexpr uint32_t kDevStatusTimeout = 2u;  // a bounded wait gave up    -> S4R_ERR_TIMEOUT

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// Number of elements of T in 16 bytes.
template <typename T> struct Vec16 { static constexpr int n = 16 / sizeof(T); };

// Load 16 bytes (n = 4 floats or 8 bf16) starting at p (16-byte aligned) as floats.
__device__ __forceinline__ void load16(const float *p, float *out) {
  const float4 v = *reinterpret_cast<const float4 *>(p);
  out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}
__device__ __forceinline__ void load16(const bf16 *p, float *out) {
  const uint4 v = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(w[i] << 16);
    out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ void set_status(uint32_t *status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Decode-step shape shared by the kernels (plain values, passed by value).
struct Shape {
  int32_t batch, n_heads_q, n_heads_kv, head_dim, rank_k, rank_v;
  int32_t n_sink, local_window, top_k, query_window, pool_kernel, pool_mode, row_mode;
  int32_t d_model, group, n_rows;  // D', G, scoring rows R
  int64_t cache_rows;
};

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
template <typename T> __host__ __device__ __forceinline__ T smin(T a, T b) { return a < b ? a : b; }
template <typename T> __host__ __device__ __forceinline__ T smax(T a, T b) { return a < b ? b : a; }

// Number of top-k candidates of a problem with L_c coefficient rows.
__device__ __forceinline__ int64_t n_candidates(int64_t L, int32_t w) {
  const int64_t c = L - w;
  return c > 0 ? c : 0;
}

// Programmatic dependent launch.  The kernels of a decode call are launched
// so that each may start while its predecessor in the stream drains.
// pdl_wait blocks until the preceding grid has completed and its writes are
// visible; a kernel calls it before touching anything that grid (or any
// earlier work) may still write.  pdl_trigger, called after the wait, lets
// the next grid start its own prologue.  Both are no-ops for a kernel that
// was launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Level-0 bins of the candidate scores of a problem for the top-k search.
// The scores of a problem sum to its number of scoring rows R (each row's
// softmax sums to 1), so their mean is R / L_c.  A score's bin is its IEEE
// bit pattern (which orders non-negative floats like their values) minus
// that of the mean, in steps of 2^15 (1/256 of a binade), offset by
// kExpBins / 2 and clamped to [0, kExpBins): monotone in the score, fine
// around the mean, and the two edge bins take everything beyond +-8 binades.
constexpr int kExpBins = 4096;
constexpr int kExpStep = 15;
__host__ __device__ inline uint32_t score_center(int R, int64_t L) {
  const float m = L > 0 ? (float)R / (float)L : 1.0f;
  union { float f; uint32_t u; } v;
  v.f = m;
  return v.u;
}
__host__ __device__ inline int score_bin(uint32_t key, uint32_t center) {
  const int64_t d = ((int64_t)key - (int64_t)center) >> kExpStep;   // floor for negative differences
  const int64_t b = d + kExpBins / 2;
  return (int)(b < 0 ? 0 : (b >= kExpBins ? kExpBins - 1 : b));
}
// Key range [lo, hi] of bin b.
__host__ __device__ inline void score_bin_range(int b, uint32_t center, uint32_t &lo, uint32_t &hi) {
  const int64_t base = (int64_t)center + ((int64_t)(b - kExpBins / 2) << kExpStep);
  const int64_t l = b == 0 ? 0 : base;
  const int64_t h = b == kExpBins - 1 ? 0x7fffffffLL : base + (1LL << kExpStep) - 1;
  lo = (uint32_t)(l < 0 ? 0 : (l > 0x7fffffffLL ? 0x7fffffffLL : l));
  hi = (uint32_t)(h < 0 ? 0 : (h > 0x7fffffffLL ? 0x7fffffffLL : h));
}

}  // namespace s4r
