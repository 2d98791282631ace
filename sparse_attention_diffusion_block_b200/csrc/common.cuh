// Shared device helpers of the PISA library (single translation unit build).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "pisa.h"

namespace pisa {

// Device error word: set by bounded waits and index checks, read by
// pisa_device_status().  Codes mirror pisa_status (0 = fine).
__device__ int g_error_word = 0;

__device__ __forceinline__ void raise_device_error(int code) {
  atomicCAS(&g_error_word, 0, code);
}

// Limit of the bounded mbarrier waits, in ns of the global timer (one per
// device; set by pisa_set_wait_limit, 2 s unless changed).
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;
__device__ unsigned long long g_wait_limit_ns = kDefaultWaitLimitNs;

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_float(float x);
template <> __device__ __forceinline__ float from_float<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Loads 8 consecutive elements (16 bytes for bf16, 32 for fp32) as floats.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* out) {
  uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    out[2 * e] = f.x;
    out[2 * e + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float* out) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Fixed-order block reduction (deterministic for a fixed launch shape).
// `red` must hold blockDim.x/32 floats.  Result valid in every thread.
__device__ __forceinline__ float block_sum(float x, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  x = warp_sum(x);
  __syncthreads();
  if (lane == 0) red[warp] = x;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < nw; ++w) t += red[w];
  return t;
}

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace pisa
