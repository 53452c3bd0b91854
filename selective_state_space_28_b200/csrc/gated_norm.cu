// gated_norm.cu -- the Mamba-2 mixer's gated RMS norm ("Mamba-2", nnterp
// encyclopedia: "The mixer's values", out_proj(norm(y * silu(z))), and the
// paragraph on the block's norms: the gated norm multiplies y by silu(z) and
// then normalizes over the mixer's whole width, whatever n_groups is):
//
//   g = y * silu(z),   out = g / sqrt(mean(g^2) + eps) * weight,
//
// the mean taken over a token's whole row (heads x head_dim).  The statistic
// needs every head of the token, so it is a pass of its own after the SSD.
//
// One CTA per row: the first pass reads y and z with 16-byte streaming loads
// and accumulates the sum of squares of g; a block reduction gives the row's
// scale; the second pass writes out.  Rows up to 8192 bf16 / 4096 float32
// values keep g in registers (all of a thread's loads issued before any is
// used, so enough bytes are in flight); wider rows keep it in shared memory.
// Every input is read once and every output written once.  out may be y
// itself (the whole row is read before any of it is written).
#include "common.cuh"
#include "internal.h"

namespace ssm {
namespace {

constexpr int kThreads = 256;

template <typename T> struct NVec;
template <> struct NVec<__nv_bfloat16> {
  static constexpr int V = 8;
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&f)[8]) {
    const uint4 w = __ldcs(reinterpret_cast<const uint4 *>(p));
    f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
    f[4] = bf16lo(w.z); f[5] = bf16hi(w.z); f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&f)[8]) {
    __stcs(reinterpret_cast<uint4 *>(p),
           make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7])));
  }
};
template <> struct NVec<float> {
  static constexpr int V = 4;
  static __device__ __forceinline__ void load(const float *p, float (&f)[4]) {
    const float4 v = __ldcs(reinterpret_cast<const float4 *>(p));
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  static __device__ __forceinline__ void store(float *p, const float (&f)[4]) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(f[0], f[1], f[2], f[3]));
  }
};

template <typename T> __device__ __forceinline__ float gate(float z) {
  return sizeof(T) == 2 ? silu_tanh(z) : silu(z);
}

// Sum over the CTA; every thread gets the total.
__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) t += red[w];
  return t;
}

// Raw 16-byte vectors, widened after all of a thread's loads are issued.
template <typename T> struct NRaw;
template <> struct NRaw<__nv_bfloat16> {
  using R = uint4;
  static __device__ __forceinline__ R load(const __nv_bfloat16 *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
  }
  static __device__ __forceinline__ void widen(const R &w, float (&f)[8]) {
    f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
    f[4] = bf16lo(w.z); f[5] = bf16hi(w.z); f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
  }
};
template <> struct NRaw<float> {
  using R = float4;
  static __device__ __forceinline__ R load(const float *p) {
    return __ldcs(reinterpret_cast<const float4 *>(p));
  }
  static __device__ __forceinline__ void widen(const R &v, float (&f)[4]) {
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
};
constexpr int kMaxVec = 4;  // vectors per thread the register form holds

// Register form: rows of at most kThreads * V * NV values, whole vectors.
// Every thread issues all of its (up to NV) y and z loads before using any,
// keeps its gated values in registers across the block reduction, and writes
// its outputs from them: each input read once, each output written once, no
// shared-memory copy of the row.  The launch picks the smallest NV that
// covers the row (the 2.7B mixer's 5120 bf16 values: NV = 3), so a thread
// holds no registers for vectors it never loads.
template <typename T, int NV>
__global__ void __launch_bounds__(kThreads) gated_norm_reg_kernel(GatedNormParams p) {
  constexpr int V = NVec<T>::V;
  __shared__ float red[kThreads / 32];
  const int64_t W = p.width;
  const T *y = static_cast<const T *>(p.y) + (int64_t)blockIdx.x * W;
  const T *z = p.z ? static_cast<const T *>(p.z) + (int64_t)blockIdx.x * W : nullptr;
  T *o = static_cast<T *>(p.out) + (int64_t)blockIdx.x * W;
  typename NRaw<T>::R ry[NV], rz[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = (k * kThreads + (int)threadIdx.x) * V;
    if (i < W) {
      ry[k] = NRaw<T>::load(y + i);
      if (z) rz[k] = NRaw<T>::load(z + i);
    }
  }
  float g[NV][V];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = (k * kThreads + (int)threadIdx.x) * V;
    if (i < W) {
      float yv[V], zv[V];
      NRaw<T>::widen(ry[k], yv);
      if (z) NRaw<T>::widen(rz[k], zv);
#pragma unroll
      for (int v = 0; v < V; ++v) {
        g[k][v] = z ? yv[v] * gate<T>(zv[v]) : yv[v];
        ss = fmaf(g[k][v], g[k][v], ss);
      }
    }
  }
  const float inv = rsqrtf(block_sum(ss, red) / (float)W + p.eps);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = (k * kThreads + (int)threadIdx.x) * V;
    if (i < W) {
      float ov[V];
#pragma unroll
      for (int v = 0; v < V; v += 4) {
        float4 wq = make_float4(1.f, 1.f, 1.f, 1.f);
        if (p.weight) wq = *reinterpret_cast<const float4 *>(p.weight + i + v);
        ov[v] = g[k][v] * inv * wq.x;
        ov[v + 1] = g[k][v + 1] * inv * wq.y;
        ov[v + 2] = g[k][v + 2] * inv * wq.z;
        ov[v + 3] = g[k][v + 3] * inv * wq.w;
      }
      NVec<T>::store(o + i, ov);
    }
  }
}

// Shared-memory form, for wider rows (VEC: whole 16-byte vectors) and for
// rows that are not whole vectors (!VEC): the gated row is kept in shared
// memory between the two passes.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads) gated_norm_kernel(GatedNormParams p) {
  extern __shared__ float4 g4[];  // [width]: this row's gated values
  float *g = reinterpret_cast<float *>(g4);
  __shared__ float red[kThreads / 32];
  const int64_t W = p.width;
  const T *y = static_cast<const T *>(p.y) + (int64_t)blockIdx.x * W;
  const T *z = p.z ? static_cast<const T *>(p.z) + (int64_t)blockIdx.x * W : nullptr;
  T *o = static_cast<T *>(p.out) + (int64_t)blockIdx.x * W;
  float ss = 0.f;
  if constexpr (VEC) {
    constexpr int V = NVec<T>::V;
    for (int64_t i = (int64_t)threadIdx.x * V; i < W; i += (int64_t)kThreads * V) {
      float yv[V], zv[V];
      NVec<T>::load(y + i, yv);
      if (z) NVec<T>::load(z + i, zv);
      float gv[V];
#pragma unroll
      for (int v = 0; v < V; ++v) {
        gv[v] = z ? yv[v] * gate<T>(zv[v]) : yv[v];
        ss = fmaf(gv[v], gv[v], ss);
      }
#pragma unroll
      for (int v = 0; v < V; v += 4)
        *reinterpret_cast<float4 *>(&g[i + v]) = make_float4(gv[v], gv[v + 1], gv[v + 2], gv[v + 3]);
    }
  } else {
    for (int64_t i = threadIdx.x; i < W; i += kThreads) {
      const float yv = ld(y + i);
      const float gv = z ? yv * gate<T>(ld(z + i)) : yv;
      g[i] = gv;
      ss = fmaf(gv, gv, ss);
    }
  }
  const float inv = rsqrtf(block_sum(ss, red) / (float)W + p.eps);
  // (block_sum's barrier also orders every g[] write before the reads below)
  if constexpr (VEC) {
    constexpr int V = NVec<T>::V;
    for (int64_t i = (int64_t)threadIdx.x * V; i < W; i += (int64_t)kThreads * V) {
      float ov[V];
#pragma unroll
      for (int v = 0; v < V; v += 4) {
        const float4 gq = *reinterpret_cast<const float4 *>(&g[i + v]);
        float4 wq = make_float4(1.f, 1.f, 1.f, 1.f);
        if (p.weight) wq = *reinterpret_cast<const float4 *>(p.weight + i + v);
        ov[v] = gq.x * inv * wq.x;
        ov[v + 1] = gq.y * inv * wq.y;
        ov[v + 2] = gq.z * inv * wq.z;
        ov[v + 3] = gq.w * inv * wq.w;
      }
      NVec<T>::store(o + i, ov);
    }
  } else {
    for (int64_t i = threadIdx.x; i < W; i += kThreads)
      st(o + i, g[i] * inv * (p.weight ? p.weight[i] : 1.f));
  }
}

template <typename T>
cudaError_t launch_t(const GatedNormParams &p, cudaStream_t s) {
  constexpr int V = NVec<T>::V;
  const bool vec = (p.width % V) == 0;  // rows are then whole 16-byte vectors
  const int64_t nv = (p.width + (int64_t)kThreads * V - 1) / ((int64_t)kThreads * V);
  const unsigned grid = (unsigned)p.rows;
  if (vec && nv <= kMaxVec) {
    switch (nv) {
      case 1: gated_norm_reg_kernel<T, 1><<<grid, kThreads, 0, s>>>(p); break;
      case 2: gated_norm_reg_kernel<T, 2><<<grid, kThreads, 0, s>>>(p); break;
      case 3: gated_norm_reg_kernel<T, 3><<<grid, kThreads, 0, s>>>(p); break;
      default: gated_norm_reg_kernel<T, 4><<<grid, kThreads, 0, s>>>(p); break;
    }
    return cudaGetLastError();
  }
  const size_t smem = (size_t)p.width * sizeof(float);
  auto kern = vec ? gated_norm_kernel<T, true> : gated_norm_kernel<T, false>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool gated_norm_supported(const GatedNormParams &p) {
  return p.width >= 1 && p.width <= kGatedNormMaxWidth && p.rows < (1ll << 31);
}

cudaError_t launch_gated_norm(const GatedNormParams &p, cudaStream_t s) {
  return p.io == 1 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace ssm
