// scan_m1.cu -- Mamba-1 selective scan (kernel a): the generic form, used for
// shapes the pipelined form (scan_m1_tma.cu) cannot tile, and the pre-pass
// for the step-input RMS norm.
//
// Computes, per batch b, channel c and token t ("Mamba", nnterp guide, intro
// and "The values"; "Mamba", tokentrails, "Code"):
//   d = softplus(dt * rstd + dt_bias[c]);  h[n] = exp(d A[c,n]) h[n] + d B[n] x
//   y = C . h + D[c] x;  y *= silu(z)
//
// Work split.  One CTA owns one batch row and a tile of 32 channels for the
// whole sequence, so the recurrence never leaves the CTA and needs no
// inter-CTA wait.  Each channel's N states are spread over N/4 lanes (4
// states per lane, fp32, in registers).  The sequence is walked in stages of
// 32 tokens: all threads first stage the step, step*x, x and z of the stage
// in shared memory (the per-element prologue runs once per element, not once
// per lane), then every lane advances its 4 states through the stage and
// the N/4 lanes of a channel combine their partial C.h with warp shuffles,
// then all threads apply the D*x skip and the gate and store y.
#include "common.cuh"
#include "internal.h"

namespace ssm {
namespace {

constexpr int kCT = 32;  // channels per CTA
constexpr int kTL = 32;  // tokens per stage

template <int N, typename T, bool HAS_Z, bool STATES>
__global__ void __launch_bounds__(kCT *(N / 4))
    m1_scan_kernel(const M1Params p) {
  constexpr int LPC = N / 4;  // lanes per channel
  constexpr int NT = kCT * LPC;
  __shared__ float sd[kTL][kCT], sdx[kTL][kCT], sx[kTL][kCT], sz[kTL][kCT],
      sy[kTL][kCT];
  __shared__ __align__(16) float sB[kTL][N];
  __shared__ __align__(16) float sC[kTL][N];
  __shared__ float srow[kTL][2];

  const int64_t L = p.L, C = p.C, G = p.G;
  const int b = blockIdx.y;
  const int64_t c0 = (int64_t)blockIdx.x * kCT;
  const int tid = threadIdx.x;
  const int cl = tid / LPC, q = tid % LPC;
  const int64_t c = c0 + cl;
  const bool cvalid = c < C;
  const int64_t g = c0 / (C / G);  // the whole tile lies in one group
  const T *x = static_cast<const T *>(p.x);
  const T *dt = static_cast<const T *>(p.dt);
  const T *z = static_cast<const T *>(p.z);
  const T *Bp = static_cast<const T *>(p.B);
  const T *Cp = static_cast<const T *>(p.Cm);
  T *y = static_cast<T *>(p.y);
  const bool softplus_on = p.flags & 1u;
  const bool rms_bc = p.flags & 2u;

  float h[4], Al[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    h[j] = (cvalid && p.h0) ? p.h0[(b * C + c) * N + 4 * q + j] : 0.f;
    Al[j] = cvalid ? p.A[c * N + 4 * q + j] * kLog2e : 0.f;
  }

  for (int64_t t0 = 0; t0 < L; t0 += kTL) {
    const int tn = (int)(L - t0 < kTL ? L - t0 : kTL);
    // ---- stage: per-element prologue, once per (token, channel)
    for (int e = tid; e < kTL * kCT; e += NT) {
      const int t = e / kCT, cc = e % kCT;
      const int64_t cg = c0 + cc;
      float dv = 0.f, xv = 0.f, zv = 0.f;
      if (t < tn && cg < C) {
        const int64_t i = (b * L + t0 + t) * C + cg;
        xv = ld(x + i);
        dv = ld(dt + i);
        if (p.rstd) dv *= p.rstd[b * L + t0 + t];
        if (p.dt_bias) dv += p.dt_bias[cg];
        if (softplus_on) dv = softplus(dv);
        if (HAS_Z) zv = ld(z + i);
      }
      sd[t][cc] = dv;
      sdx[t][cc] = dv * xv;
      sx[t][cc] = xv;
      sz[t][cc] = zv;
    }
    for (int e = tid; e < kTL * N; e += NT) {
      const int t = e / N, n = e % N;
      float bv = 0.f, cv = 0.f;
      if (t < tn) {
        const int64_t i = ((b * L + t0 + t) * G + g) * N + n;
        bv = ld(Bp + i);
        cv = ld(Cp + i);
      }
      sB[t][n] = bv;
      sC[t][n] = cv;
    }
    __syncthreads();
    if (rms_bc) {  // weightless RMS norm of each token's B and C over N
      for (int e = tid; e < kTL * 2; e += NT) {
        const int t = e / 2;
        const float *row = (e & 1) ? sC[t] : sB[t];
        float ss = 0.f;
#pragma unroll
        for (int n = 0; n < N; ++n) ss += row[n] * row[n];
        srow[t][e & 1] = rsqrtf(ss / N + p.eps);
      }
      __syncthreads();
      for (int e = tid; e < kTL * N; e += NT) {
        const int t = e / N, n = e % N;
        sB[t][n] *= srow[t][0];
        sC[t][n] *= srow[t][1];
      }
      __syncthreads();
    }
    // ---- recurrence over the stage: 4 states per lane
    for (int t = 0; t < tn; ++t) {
      const float d = sd[t][cl], dx = sdx[t][cl];
      const float4 b4 = *reinterpret_cast<const float4 *>(&sB[t][4 * q]);
      const float4 c4 = *reinterpret_cast<const float4 *>(&sC[t][4 * q]);
      h[0] = ex2(d * Al[0]) * h[0] + dx * b4.x;
      h[1] = ex2(d * Al[1]) * h[1] + dx * b4.y;
      h[2] = ex2(d * Al[2]) * h[2] + dx * b4.z;
      h[3] = ex2(d * Al[3]) * h[3] + dx * b4.w;
      if (p.state_write && t0 + t == p.t_write && cvalid) {
        // a state written at this token replaces h_t: y_t reads it and the
        // tokens after continue from it ("Mamba", nnterp guide, "The state")
        const float4 w4 =
            *reinterpret_cast<const float4 *>(p.state_write + (b * C + c) * N + 4 * q);
        h[0] = w4.x; h[1] = w4.y; h[2] = w4.z; h[3] = w4.w;
      }
      float acc = c4.x * h[0] + c4.y * h[1] + c4.z * h[2] + c4.w * h[3];
#pragma unroll
      for (int off = LPC / 2; off > 0; off >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (q == 0) sy[t][cl] = acc;
      if (STATES && cvalid)
        *reinterpret_cast<float4 *>(p.states + ((b * L + t0 + t) * C + c) * N + 4 * q) =
            make_float4(h[0], h[1], h[2], h[3]);
    }
    __syncthreads();
    // ---- epilogue: skip term, gate, store
    for (int e = tid; e < kTL * kCT; e += NT) {
      const int t = e / kCT, cc = e % kCT;
      const int64_t cg = c0 + cc;
      if (t < tn && cg < C) {
        float yv = sy[t][cc] + (p.D ? p.D[cg] : 0.f) * sx[t][cc];
        if (HAS_Z) yv *= silu(sz[t][cc]);
        st(y + (b * L + t0 + t) * C + cg, yv);
      }
    }
    __syncthreads();
  }
  if (p.h_last && cvalid)
    *reinterpret_cast<float4 *>(p.h_last + (b * C + c) * N + 4 * q) =
        make_float4(h[0], h[1], h[2], h[3]);
}

// Sum of squares of the values in one 16-byte vector of the I/O type.
__device__ __forceinline__ float sumsq16(const uint4 &w, const __nv_bfloat16 *) {
  float s = 0.f;
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = bf16lo(u[i]), b = bf16hi(u[i]);
    s = fmaf(a, a, s);
    s = fmaf(b, b, s);
  }
  return s;
}
__device__ __forceinline__ float sumsq16(const uint4 &w, const float *) {
  const float a = __uint_as_float(w.x), b = __uint_as_float(w.y), c = __uint_as_float(w.z),
              d = __uint_as_float(w.w);
  return fmaf(a, a, fmaf(b, b, fmaf(c, c, d * d)));
}

// Per (batch, token) RMS factor of the step input over the channels:
// rstd = 1 / sqrt(mean_c(dt^2) + eps).  One warp per row.  Rows of whole
// 16-byte vectors (the base is 16-byte aligned) are read a vector per lane,
// four vectors in flight per lane, so that the pass streams at the HBM rate
// rather than at the rate of 2-byte load instructions; other rows value by
// value.
template <typename T>
__global__ void dt_rms_kernel(const T *__restrict__ dt, int64_t rows, int64_t C,
                              float eps, float *__restrict__ rstd) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const T *r = dt + row * C;
  float ss = 0.f;
  constexpr int V = 16 / (int)sizeof(T);  // values per vector
  if (C % V == 0) {
    const uint4 *r4 = reinterpret_cast<const uint4 *>(r);
    const int64_t nv = C / V;
    int64_t i = lane;
    for (; i + 96 < nv; i += 128) {
      const uint4 a = r4[i], b = r4[i + 32], c = r4[i + 64], d = r4[i + 96];
      ss += (sumsq16(a, r) + sumsq16(b, r)) + (sumsq16(c, r) + sumsq16(d, r));
    }
    for (; i < nv; i += 32) ss += sumsq16(r4[i], r);
  } else {
    for (int64_t c = lane; c < C; c += 32) {
      const float v = ld(r + c);
      ss += v * v;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (lane == 0) rstd[row] = rsqrtf(ss / (float)C + eps);
}

template <int N, typename T>
cudaError_t launch_n(const M1Params &p, cudaStream_t s) {
  dim3 grid((unsigned)((p.C + kCT - 1) / kCT), (unsigned)p.batch);
  dim3 block(kCT * (N / 4));
  const bool hz = p.z != nullptr, hs = p.states != nullptr;
  if (hz && hs) m1_scan_kernel<N, T, true, true><<<grid, block, 0, s>>>(p);
  else if (hz) m1_scan_kernel<N, T, true, false><<<grid, block, 0, s>>>(p);
  else if (hs) m1_scan_kernel<N, T, false, true><<<grid, block, 0, s>>>(p);
  else m1_scan_kernel<N, T, false, false><<<grid, block, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const M1Params &p, cudaStream_t s) {
  if (p.rstd) {
    const int64_t rows = p.batch * p.L;
    dt_rms_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
        static_cast<const T *>(p.dt), rows, p.C, p.eps, p.rstd);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // the pipelined kernel wherever the shape allows; a state write together
  // with per-token states takes the generic kernel
  if (!(p.state_write && p.states) && m1_scan_tma_supported(p)) return launch_m1_scan_tma(p, s);
  switch (p.N) {
    case 4: return launch_n<4, T>(p, s);
    case 8: return launch_n<8, T>(p, s);
    case 16: return launch_n<16, T>(p, s);
    case 32: return launch_n<32, T>(p, s);
    case 64: return launch_n<64, T>(p, s);
  }
  return cudaErrorNotSupported;
}

}  // namespace

bool m1_scan_supported(int64_t N, int64_t C, int64_t G) {
  const bool n_ok = N == 4 || N == 8 || N == 16 || N == 32 || N == 64;
  const bool g_ok = G == 1 || ((C / G) % kCT == 0);
  return n_ok && g_ok;
}

cudaError_t launch_m1_scan(const M1Params &p, cudaStream_t s) {
  if (!m1_scan_supported(p.N, p.C, p.G)) return cudaErrorNotSupported;
  if (p.batch == 0 || p.L == 0) return cudaSuccess;
  return p.io == 1 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace ssm
