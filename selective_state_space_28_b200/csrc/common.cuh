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

// silu(z) = z * sigmoid(z) = z * (1 + tanh(z / 2)) / 2, with the SFU's
// tanh.approx.f32 (one SFU operation instead of ex2 and a reciprocal).  Its
// absolute error is a few 2^-11 of z: enough for bfloat16 outputs.
__device__ __forceinline__ float silu_tanh(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  return z * fmaf(0.5f, t, 0.5f);
}

// ------------------------------------------------------------ packed f32x2

struct f2 {
  float x, y;
};
__device__ __forceinline__ f2 mk2(float a, float b) { return {a, b}; }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
  f2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// softplus(v) = log(1 + e^v), float32, from the SFU's ex2/lg2: for e^v < 1/32
// a 4-term series of log1p (relative error below 2e-7), above it lg2(1 + e^v)
// (the rounding of 1 + e^v then costs at most 2 ulp relative); v > 20 gives v.
__device__ __forceinline__ float softplus_sfu(float v) {
  const float u = ex2(v * kLog2e);
  float lg;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(1.f + u));
  const float series = u * fmaf(u, fmaf(u, fmaf(u, -0.25f, 0.33333334f), -0.5f), 1.f);
  const float r = u < 0.03125f ? series : lg * 0.6931471806f;
  return v > 20.f ? v : r;
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
