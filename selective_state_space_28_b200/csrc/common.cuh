// common.cuh -- small device helpers shared by the libssm kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// log2(e): exp(v) = 2^(v * log2(e)).
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- I/O types

template <typename T> struct IO;
template <> struct IO<float> {
  static __device__ __forceinline__ float load(const float *p) { return *p; }
  static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
};
template <> struct IO<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) {
    *p = __float2bfloat16_rn(v);
  }
};

template <typename T> __device__ __forceinline__ float ld(const T *p) { return IO<T>::load(p); }
template <typename T> __device__ __forceinline__ void st(T *p, float v) { IO<T>::store(p, v); }

// bf16 -> f32 is exact: the bf16 bits are the top half of the f32 bits.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two f32 -> packed bf16x2, round to nearest even (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ------------------------------------------------------------ elementwise

// 2^v with the SFU's approximate exponential (ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// softplus(v) = log(1 + e^v).  Above 20 the correction e^-v is below half an
// ulp of v in float32, so v itself is returned.  softplus(-inf) = 0 exactly.
__device__ __forceinline__ float softplus(float v) {
  return v > 20.f ? v : log1pf(ex2(v * kLog2e));
}

// silu(z) = z * sigmoid(z) = z / (1 + e^-z).
__device__ __forceinline__ float silu(float z) {
  return z / (1.f + ex2(-z * kLog2e));
}

// --------------------------------------------------------- cache hints

// Streaming 16-byte load/store (no reuse expected: evict-first).
__device__ __forceinline__ float4 ld_stream4(const float4 *p) {
  float4 r;
  asm volatile("ld.global.cs.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ void st_stream4(float4 *p, float4 v) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

}  // namespace ssm
