// Shared device helpers for the retention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "retention.h"

namespace ret {

// Element access for the two storage types of q, k, v, o.
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float x) { *p = x; }
  // four consecutive elements (16-byte aligned address)
  static __device__ __forceinline__ float4 ld4(const float* p) {
    return *reinterpret_cast<const float4*>(p);
  }
  static __device__ __forceinline__ void st4(float* p, float4 x) {
    *reinterpret_cast<float4*>(p) = x;
  }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
  // four consecutive elements (8-byte aligned address)
  static __device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    float4 r;
    r.x = __uint_as_float(u.x << 16);
    r.y = __uint_as_float(u.x & 0xffff0000u);
    r.z = __uint_as_float(u.y << 16);
    r.w = __uint_as_float(u.y & 0xffff0000u);
    return r;
  }
  static __device__ __forceinline__ void st4(__nv_bfloat16* p, float4 x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  }
};

// gamma^n for an integer n >= 0, given lg = log2(gamma).  n == 0 gives 1 for
// every gamma (0^0 = 1); gamma == 0 has lg = -inf and gives 0 for n > 0.
__device__ __forceinline__ float gpow(float lg, int n) {
  return n == 0 ? 1.0f : exp2f(static_cast<float>(n) * lg);
}

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// swish(x) = x sigmoid(x) = x / (1 + e^-x), the activation of the output
// gate; e^-x overflows to inf for very negative x, which gives -0.
__device__ __forceinline__ float swishf(float x) { return x / (1.0f + __expf(-x)); }

}  // namespace ret
