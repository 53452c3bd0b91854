// step.cu -- the decode step (kernel c) and the Mamba-2 token recurrence.
//
// Mamba-2 ("Mamba-2", nnterp encyclopedia, "The mixer's values", "The
// state"): per (batch, head) an N x P float32 state, key side first.  Each
// token decays the whole state by one scalar a = exp(d A_h) and adds the
// outer product d B x^T; y = C^T h + D x, read AFTER the update ("Mamba",
// nnterp guide, "Read order on a decode step").
//
// One CTA owns one (batch, head).  Thread (rg, pq) holds the state rows
// n = rg + k*RS (k < K) at the four value columns 4pq..4pq+3 as float4
// registers, so the state is read once and written once with 16-byte
// accesses.  Tokens are staged TT at a time in shared memory; the y partial
// sums over the RS row groups are reduced through shared memory once per
// stage.  With L = 1 and h0 == h_last == the cached state this is the decode
// step, updating the state in place (each thread rewrites exactly what it
// read).
//
// Mamba-1 step: one token against a [batch, C, N] state; 4 states per lane,
// N/4 lanes per channel, y combined with warp shuffles.
#include "common.cuh"
#include "internal.h"

namespace ssm {
namespace {

// Row of the k-th state row a lane of the P = 64 step kernel owns: blocks of
// 8 consecutive rows, the next block 128 rows further on.
__device__ __forceinline__ int rowof(int n0, int k) { return n0 + (k & 7) + 128 * (k >> 3); }

template <typename T, bool HAS_Z, int K, int TT>
__global__ void __launch_bounds__(256) m2_recurrent_kernel(const M2Params p) {
  extern __shared__ __align__(16) float smem[];
  const int64_t L = p.L, H = p.H, P = p.P, N = p.N, G = p.G;
  const int P4 = (int)(P / 4);
  const int RS = (int)(N / K);
  const int NT = P4 * RS;
  const int tid = threadIdx.x;
  const int pq = tid % P4, rg = tid / P4;
  const int64_t hd = blockIdx.x, b = blockIdx.y;
  const int64_t g = hd / (H / G);
  const int64_t TN4 = (TT * N + 3) & ~3;  // keeps every array 16-byte aligned
  float *sx = smem;                 // [TT][P]
  float *sB = sx + TT * P;          // [TT][N]  (B * d)
  float *sC = sB + TN4;             // [TT][N]
  float *sa = sC + TN4;             // [TT]     decay exp(d A)
  float *sd = sa + TT;              // [TT]     step d
  float *ys = sa + 2 * ((TT + 3) & ~3); // [TT][RS][P]
  const T *x = static_cast<const T *>(p.x);
  const T *z = static_cast<const T *>(p.z);
  const T *dt = static_cast<const T *>(p.dt);
  const T *Bp = static_cast<const T *>(p.B);
  const T *Cp = static_cast<const T *>(p.Cm);
  T *y = static_cast<T *>(p.y);
  const float A2 = p.A[hd] * kLog2e;
  const float bias = p.dt_bias ? p.dt_bias[hd] : 0.f;
  const float Dh = p.D ? p.D[hd] : 0.f;
  const bool softplus_on = p.flags & 1u;

  float4 S[K];
  const int64_t sbase = (b * H + hd) * N * P;
#pragma unroll
  for (int k = 0; k < K; ++k)
    S[k] = p.h0 ? *reinterpret_cast<const float4 *>(p.h0 + sbase + (rg + k * RS) * P + 4 * pq)
                : make_float4(0.f, 0.f, 0.f, 0.f);

  for (int64_t t0 = 0; t0 < L; t0 += TT) {
    const int tn = (int)(L - t0 < TT ? L - t0 : TT);
    for (int e = tid; e < tn; e += NT) {
      float d = ld(dt + (b * L + t0 + e) * H + hd) + bias;
      if (softplus_on) d = softplus(d);
      sa[e] = ex2(d * A2);
      sd[e] = d;
    }
    __syncthreads();
    for (int e = tid; e < tn * N; e += NT) {
      const int t = e / (int)N, n = e % (int)N;
      const int64_t i = ((b * L + t0 + t) * G + g) * N + n;
      sB[e] = ld(Bp + i) * sd[t];
      sC[e] = ld(Cp + i);
    }
    for (int e = tid; e < tn * P; e += NT) {
      const int t = e / (int)P, c = e % (int)P;
      sx[e] = ld(x + ((b * L + t0 + t) * H + hd) * P + c);
    }
    __syncthreads();
    for (int t = 0; t < tn; ++t) {
      const float a = sa[t];
      const float4 xq = *reinterpret_cast<const float4 *>(sx + t * P + 4 * pq);
      float4 yp = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const float bn = sB[t * N + rg + k * RS];
        const float cn = sC[t * N + rg + k * RS];
        S[k].x = a * S[k].x + bn * xq.x;
        S[k].y = a * S[k].y + bn * xq.y;
        S[k].z = a * S[k].z + bn * xq.z;
        S[k].w = a * S[k].w + bn * xq.w;
        yp.x += cn * S[k].x;
        yp.y += cn * S[k].y;
        yp.z += cn * S[k].z;
        yp.w += cn * S[k].w;
      }
      if (p.states) {
        float *sp = p.states + ((b * L + t0 + t) * H + hd) * N * P;
#pragma unroll
        for (int k = 0; k < K; ++k)
          *reinterpret_cast<float4 *>(sp + (rg + k * RS) * P + 4 * pq) = S[k];
      }
      *reinterpret_cast<float4 *>(ys + ((int64_t)t * RS + rg) * P + 4 * pq) = yp;
    }
    __syncthreads();
    for (int e = tid; e < tn * P; e += NT) {
      const int t = e / (int)P, c = e % (int)P;
      float acc = 0.f;
      for (int r = 0; r < RS; ++r) acc += ys[((int64_t)t * RS + r) * P + c];
      const int64_t i = ((b * L + t0 + t) * H + hd) * P + c;
      float yv = acc + Dh * sx[e];
      if (HAS_Z) yv *= silu(ld(z + i));
      st(y + i, yv);
    }
    __syncthreads();
  }
  if (p.h_last) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      *reinterpret_cast<float4 *>(p.h_last + sbase + (rg + k * RS) * P + 4 * pq) = S[k];
  }
}

// Threads = (P/4) * RS with RS = N / K rows per pass, at most 256.
bool m2_shape(int64_t N, int64_t P, int *K_out, int *RS_out) {
  if (P % 4 || P < 4 || N < 1) return false;
  const int64_t P4 = P / 4;
  if (P4 > 256 || 256 % P4) return false;
  int64_t RS = 256 / P4;
  if (RS > N) RS = N;
  if (N % RS) return false;
  const int64_t K = N / RS;
  if (K != 1 && K != 2 && K != 4 && K != 8 && K != 16) return false;
  *K_out = (int)K;
  *RS_out = (int)RS;
  return true;
}

template <typename T, bool HZ, int K>
cudaError_t launch_m2_k(const M2Params &p, int RS, cudaStream_t s) {
  const int TT = p.L == 1 ? 1 : 8;
  const int64_t P = p.P, N = p.N;
  const size_t smem =
      sizeof(float) * (TT * P + 2 * ((TT * N + 3) & ~3) + 2 * ((TT + 3) & ~3) +
                       (size_t)TT * RS * P);
  dim3 grid((unsigned)p.H, (unsigned)p.batch);
  dim3 block((unsigned)(P / 4 * RS));
  if (TT == 1) {
    auto k = m2_recurrent_kernel<T, HZ, K, 1>;
    if (smem > 48 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    k<<<grid, block, smem, s>>>(p);
  } else {
    auto k = m2_recurrent_kernel<T, HZ, K, 8>;
    if (smem > 48 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    k<<<grid, block, smem, s>>>(p);
  }
  return cudaGetLastError();
}

template <typename T, bool HZ>
cudaError_t launch_m2_t(const M2Params &p, int K, int RS, cudaStream_t s) {
  switch (K) {
    case 1: return launch_m2_k<T, HZ, 1>(p, RS, s);
    case 2: return launch_m2_k<T, HZ, 2>(p, RS, s);
    case 4: return launch_m2_k<T, HZ, 4>(p, RS, s);
    case 8: return launch_m2_k<T, HZ, 8>(p, RS, s);
    case 16: return launch_m2_k<T, HZ, 16>(p, RS, s);
  }
  return cudaErrorNotSupported;
}

// ------------------------------------------------- Mamba-2 step, P = 64

// One decode token for one (batch, head) per CTA of 256 threads, head dim 64,
// state N = 16 * K.  Lane l of warp w owns the four value columns 4(l%16)..+3
// of the K rows n = 16 w + 8 (l / 16) + k: each float4 load/store of a warp
// covers two 256-byte row segments.  The token's inputs are read straight
// from global memory (B and C rows as one 16-byte load per lane), so the only
// barrier is the one that combines the eight warps' partial C^T h.
template <typename T, bool HAS_Z, int K>
__global__ void __launch_bounds__(256, 3) m2_step_kernel(const M2Params p) {
  constexpr int kP = 64;
  constexpr int N = 16 * K;
  __shared__ float4 ys[8][16];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pq = lane & 15, half = lane >> 4;
  const int64_t hd = blockIdx.x, b = blockIdx.y;
  const int64_t H = p.H, G = p.G;
  const int64_t g = hd / (H / G);
  const int n0 = 16 * warp + 8 * half;  // rows rowof(n0, k), k < K
  float *state = const_cast<float *>(p.h0) + (b * H + hd) * (int64_t)N * kP;

  // State first: every load in flight before any arithmetic.
  float4 S[K];
#pragma unroll
  for (int k = 0; k < K; ++k)
    S[k] = ld_stream4(reinterpret_cast<const float4 *>(state + (int64_t)(rowof(n0, k)) * kP + 4 * pq));

  const T *Bp = static_cast<const T *>(p.B) + (b * G + g) * N;
  const T *Cp = static_cast<const T *>(p.Cm) + (b * G + g) * N;
  float bn[K], cn[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    bn[k] = ld(Bp + rowof(n0, k));
    cn[k] = ld(Cp + rowof(n0, k));
  }
  const T *xp = static_cast<const T *>(p.x) + (b * H + hd) * kP + 4 * pq;
  const float4 xq = make_float4(ld(xp), ld(xp + 1), ld(xp + 2), ld(xp + 3));
  float d = ld(static_cast<const T *>(p.dt) + b * H + hd) + (p.dt_bias ? p.dt_bias[hd] : 0.f);
  if (p.flags & 1u) d = softplus(d);
  const float a = ex2(d * (p.A[hd] * kLog2e));

  float4 yp = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const float w = d * bn[k];
    S[k].x = a * S[k].x + w * xq.x;
    S[k].y = a * S[k].y + w * xq.y;
    S[k].z = a * S[k].z + w * xq.z;
    S[k].w = a * S[k].w + w * xq.w;
    yp.x += cn[k] * S[k].x;
    yp.y += cn[k] * S[k].y;
    yp.z += cn[k] * S[k].z;
    yp.w += cn[k] * S[k].w;
  }
#pragma unroll
  for (int k = 0; k < K; ++k)
    st_stream4(reinterpret_cast<float4 *>(state + (int64_t)(rowof(n0, k)) * kP + 4 * pq), S[k]);
  yp.x += __shfl_xor_sync(0xffffffffu, yp.x, 16);
  yp.y += __shfl_xor_sync(0xffffffffu, yp.y, 16);
  yp.z += __shfl_xor_sync(0xffffffffu, yp.z, 16);
  yp.w += __shfl_xor_sync(0xffffffffu, yp.w, 16);
  if (half == 0) ys[warp][pq] = yp;
  __syncthreads();
  if (tid < 16) {
    float4 acc = ys[0][tid];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
      const float4 v = ys[w][tid];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    const float Dh = p.D ? p.D[hd] : 0.f;
    const T *xr = static_cast<const T *>(p.x) + (b * H + hd) * kP + 4 * tid;
    float o[4] = {acc.x + Dh * ld(xr), acc.y + Dh * ld(xr + 1), acc.z + Dh * ld(xr + 2),
                  acc.w + Dh * ld(xr + 3)};
    T *yo = static_cast<T *>(p.y) + (b * H + hd) * kP + 4 * tid;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (HAS_Z) o[j] *= silu(ld(static_cast<const T *>(p.z) + (b * H + hd) * kP + 4 * tid + j));
      st(yo + j, o[j]);
    }
  }
}

// ------------------------------------------------------------ Mamba-1 step

template <int N, typename T, bool HAS_Z>
__global__ void __launch_bounds__(256) m1_step_kernel(const M1StepParams p) {
  constexpr int LPC = N / 4;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t unit = gid / LPC;  // b * C + c
  const int q = (int)(gid % LPC);
  const bool valid = unit < p.batch * p.C;
  const int64_t u = valid ? unit : 0;
  const int64_t b = u / p.C, c = u % p.C;
  const int64_t g = c / (p.C / p.G);
  const T *x = static_cast<const T *>(p.x);
  const T *dt = static_cast<const T *>(p.dt);
  const T *Bp = static_cast<const T *>(p.B);
  const T *Cp = static_cast<const T *>(p.Cm);

  float d = ld(dt + u);
  if (p.dt_bias) d += p.dt_bias[c];
  if (p.flags & 1u) d = softplus(d);
  const float xv = ld(x + u);
  float bv[4], cv[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    bv[j] = ld(Bp + (b * p.G + g) * N + 4 * q + j);
    cv[j] = ld(Cp + (b * p.G + g) * N + 4 * q + j);
  }
  if (p.flags & 2u) {  // weightless RMS norm of B and C over N
    float sb = 0.f, sc = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sb += bv[j] * bv[j];
      sc += cv[j] * cv[j];
    }
#pragma unroll
    for (int off = LPC / 2; off > 0; off >>= 1) {
      sb += __shfl_xor_sync(0xffffffffu, sb, off);
      sc += __shfl_xor_sync(0xffffffffu, sc, off);
    }
    const float rb = rsqrtf(sb / N + p.eps), rc = rsqrtf(sc / N + p.eps);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      bv[j] *= rb;
      cv[j] *= rc;
    }
  }
  float4 *sp = reinterpret_cast<float4 *>(p.state + u * N + 4 * q);
  float4 h = valid ? *sp : make_float4(0.f, 0.f, 0.f, 0.f);
  const float *A = p.A + c * N + 4 * q;
  const float dx = d * xv;
  h.x = ex2(d * (A[0] * kLog2e)) * h.x + dx * bv[0];
  h.y = ex2(d * (A[1] * kLog2e)) * h.y + dx * bv[1];
  h.z = ex2(d * (A[2] * kLog2e)) * h.z + dx * bv[2];
  h.w = ex2(d * (A[3] * kLog2e)) * h.w + dx * bv[3];
  float acc = cv[0] * h.x + cv[1] * h.y + cv[2] * h.z + cv[3] * h.w;
#pragma unroll
  for (int off = LPC / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (!valid) return;
  *sp = h;
  if (q == 0) {
    float yv = acc + (p.D ? p.D[c] : 0.f) * xv;
    if (HAS_Z) yv *= silu(ld(static_cast<const T *>(p.z) + u));
    st(static_cast<T *>(p.y) + u, yv);
  }
}

template <int N, typename T>
cudaError_t launch_m1_step_n(const M1StepParams &p, cudaStream_t s) {
  const int64_t threads = p.batch * p.C * (N / 4);
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  if (p.z) m1_step_kernel<N, T, true><<<blocks, 256, 0, s>>>(p);
  else m1_step_kernel<N, T, false><<<blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_m1_step_t(const M1StepParams &p, cudaStream_t s) {
  switch (p.N) {
    case 4: return launch_m1_step_n<4, T>(p, s);
    case 8: return launch_m1_step_n<8, T>(p, s);
    case 16: return launch_m1_step_n<16, T>(p, s);
    case 32: return launch_m1_step_n<32, T>(p, s);
    case 64: return launch_m1_step_n<64, T>(p, s);
  }
  return cudaErrorNotSupported;
}

}  // namespace

bool m2_recurrent_supported(int64_t N, int64_t P) {
  int K, RS;
  return m2_shape(N, P, &K, &RS);
}

cudaError_t launch_m2_recurrent(const M2Params &p, cudaStream_t s) {
  int K, RS;
  if (!m2_shape(p.N, p.P, &K, &RS)) return cudaErrorNotSupported;
  if (p.batch == 0 || p.L == 0) return cudaSuccess;
  // The decode step (one token, state updated in place) with head dim 64 and
  // state 128 has its own kernel.
  if (p.L == 1 && p.P == 64 && p.N == 128 && p.states == nullptr && p.h0 != nullptr &&
      p.h0 == p.h_last) {
    dim3 grid((unsigned)p.H, (unsigned)p.batch);
    const bool hz = p.z != nullptr;
    if (p.io == 1)
      hz ? m2_step_kernel<__nv_bfloat16, true, 8><<<grid, 256, 0, s>>>(p)
         : m2_step_kernel<__nv_bfloat16, false, 8><<<grid, 256, 0, s>>>(p);
    else
      hz ? m2_step_kernel<float, true, 8><<<grid, 256, 0, s>>>(p)
         : m2_step_kernel<float, false, 8><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
  }
  const bool hz = p.z != nullptr;
  if (p.io == 1)
    return hz ? launch_m2_t<__nv_bfloat16, true>(p, K, RS, s)
              : launch_m2_t<__nv_bfloat16, false>(p, K, RS, s);
  return hz ? launch_m2_t<float, true>(p, K, RS, s) : launch_m2_t<float, false>(p, K, RS, s);
}

bool m1_step_supported(int64_t N) {
  return N == 4 || N == 8 || N == 16 || N == 32 || N == 64;
}

cudaError_t launch_m1_step(const M1StepParams &p, cudaStream_t s) {
  if (!m1_step_supported(p.N)) return cudaErrorNotSupported;
  if (p.batch == 0) return cudaSuccess;
  return p.io == 1 ? launch_m1_step_t<__nv_bfloat16>(p, s) : launch_m1_step_t<float>(p, s);
}

}  // namespace ssm
