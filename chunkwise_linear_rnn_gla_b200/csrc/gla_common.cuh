// Device helpers shared by the kernel files.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace gla {

template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__device__ __forceinline__ void stf(T* p, float x);
template <>
__device__ __forceinline__ void stf<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

__host__ __device__ constexpr int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Floor applied to every log alpha before it enters a per-chunk cumsum. A zero gate is given as a
// huge negative log alpha (say -1e30); summed in fp32 it would swallow every later gate of the chunk
// (-1e30 + x == -1e30), losing the decay among the later steps. e^{-200} is already 0 in fp32, so
// the floor changes no factor, and sums that pass through it keep ~1e-5 relative precision.
constexpr float kLogAlphaFloor = -200.f;
__device__ __forceinline__ float la_floor(float x) { return fmaxf(x, kLogAlphaFloor); }

}  // namespace gla
