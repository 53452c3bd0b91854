// common.cuh -- small device helpers shared by the libssm kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// log2(e): exp(v) = 2^(v * log2(e)).
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------- programmatic dependent launch
// A launch made with launch_dependent() may start before the launch ahead of
// it in the stream has finished: as soon as every CTA of that launch has
// executed pdl_launch_dependents() (or exited).  Its CTAs that need the
// earlier launch's results execute pdl_wait() first, which returns once that
// launch has completed and its memory writes are visible; CTAs that need
// nothing from it run on.  In a launch made the ordinary way pdl_wait()
// returns at once.

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

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

// ------------------------------------------------- exp2 on the FMA pipe
// 2^x on the FMA pipe instead of the SFU, for decays (x = d * A2 with d >= 0
// and A2 < 0): Cody-Waite reduction 2^x = 2^j 2^f with j = round(x) and
// f = x - j in [-1/2, 1/2], a degree-5 polynomial for 2^f (coefficients and
// their weighted least-squares fit on Chebyshev nodes in gen_exp2_poly.py;
// max relative error 1.9e-7 in float32; exactly 1 at f = 0), 2^j applied
// through the exponent field.  d is first clamped to lim = -127 / A2 so that
// the exponent never drops below -127, where the result is exactly 0.

// 1.5 * 2^23 + 127: adding it rounds x to an integer j held in the low
// mantissa bits, biased by 127 so that (bits << 23) is the float 2^j.
constexpr float kMagic = 12583039.0f;
constexpr float kP1 = 6.931468844e-01f, kP2 = 2.402223796e-01f, kP3 = 5.550893024e-02f,
                kP4 = 9.671698324e-03f, kP5 = 1.321867225e-03f;

__device__ __forceinline__ f2 exp2_fma2(float d, f2 A2, f2 lim) {
  const f2 dc = mk2(fminf(d, lim.x), fminf(d, lim.y));
  const f2 t = fma2(dc, A2, mk2(kMagic, kMagic));      // j + magic
  const f2 r = add2(t, mk2(-kMagic, -kMagic));          // j
  const f2 f = fma2(dc, A2, mk2(-r.x, -r.y));           // x - j in [-1/2, 1/2]
  f2 p = fma2(mk2(kP5, kP5), f, mk2(kP4, kP4));
  p = fma2(p, f, mk2(kP3, kP3));
  p = fma2(p, f, mk2(kP2, kP2));
  p = fma2(p, f, mk2(kP1, kP1));
  p = fma2(p, f, mk2(1.f, 1.f));                        // ~ 2^f, exactly 1 at f = 0
  const f2 s = mk2(__uint_as_float(__float_as_uint(t.x) << 23),
                   __uint_as_float(__float_as_uint(t.y) << 23));  // 2^j
  return mul2(p, s);
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
