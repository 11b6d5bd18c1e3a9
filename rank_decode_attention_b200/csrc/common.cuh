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

// Bins of the histogram of the candidate scores' leading bits: the IEEE bit
// pattern of a non-negative float orders like its value, and bits 30..19
// (exponent and the top 4 mantissa bits) index 4096 bins.
constexpr int kExpBins = 4096;
constexpr int kExpShift = 19;

}  // namespace s4r
