// common.cuh -- small device helpers shared by the GDLA kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdla.h"

namespace gdla {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + __expf(-x)); }
// sigma(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh approximation (one special-function
// operation instead of an exponential and a reciprocal; relative error ~2^-11, below the
// bf16 rounding of the values it scales)
__device__ __forceinline__ float sigmoid_tanh(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

constexpr float kLog2e = 1.4426950408889634f;

// Visible(i, j): causal j <= i; sliding additionally j > i - window.
__device__ __forceinline__ bool key_visible(long i, long j, int sliding, int window) {
  return j <= i && (!sliding || j > i - window);
}

// Status word at the start of every workspace.
struct DeviceStatus {
  int code;       // gdla_status of the last call (0 = OK)
  int where;      // which wait gave up (kernel-specific tag)
  int pad[62];
};
constexpr size_t kStatusBytes = 256;

}  // namespace gdla
