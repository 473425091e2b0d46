// Shared device helpers of the HSTU CUDA path (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu.h"

namespace hstu {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------------------
// Element conversion
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// SiLU (phi1 = phi2 = SiLU, "What an HSTU layer changes") and its derivative.
// Accurate variants (expf) for the fp32 path and epilogues.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float sigmoid_acc(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float silu_acc(float x) { return x * sigmoid_acc(x); }
__device__ __forceinline__ float silu_grad_acc(float x) {
  float s = sigmoid_acc(x);
  return s * (1.0f + x * (1.0f - s));
}
// SiLU'(x) = sigma(x) (1 + x (1 - sigma(x))) with sigma(x) = (1 + tanh(x/2)) / 2,
// on the hardware tanh (relative error near 2^-11): for bf16 results.
__device__ __forceinline__ float silu_grad_fast(float x) {
  const float h = 0.5f * x;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return 0.5f * (1.f + t + fmaf(-h * t, t, h));
}
// SiLU' in the precision the element type T needs.
template <typename T> __device__ __forceinline__ float silu_grad_t(float x) { return silu_grad_acc(x); }
template <> __device__ __forceinline__ float silu_grad_t<bf16>(float x) { return silu_grad_fast(x); }

// ---------------------------------------------------------------------------
// rab^{p,t} buckets (readings: clamped linear position distance; log2 time
// gap with 0 for a zero gap).  dt is a gap in seconds, may be negative on
// masked pairs (clamped to 0).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int time_bucket(int64_t dt, int nb) {
  if (dt <= 0) return 0;
  // floor(log2 dt) + 1 == bit length of dt
  int bl = 64 - __clzll(dt);
  return bl < nb - 1 ? bl : nb - 1;
}
__device__ __forceinline__ int pos_bucket(int dp, int nb) {
  dp = dp < 0 ? 0 : dp;
  return dp < nb - 1 ? dp : nb - 1;
}

// ---------------------------------------------------------------------------
// Small reductions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace hstu
