// scan_m1_tma.cu -- Mamba-1 selective scan, pipelined form (kernel a).
//
// Same arithmetic as scan_m1.cu ("Mamba", nnterp guide, intro and "The
// values"; "Mamba", tokentrails, "Code"; "Falcon-Mamba", "Where the norms
// sit"), organised for throughput on sm_100a:
//
// * One CTA owns one batch row and CT channels for the whole sequence (the
//   recurrence never leaves the CTA).  Each channel's N states sit in
//   G = N/4 lanes, 4 float32 states per lane, in registers.
// * The sequence is walked in stages of 32 tokens.  TMA brings the stage's
//   x, dt, z ([32 x CT]) and B, C ([32 x N]) tiles into a double buffer, so
//   the loads of stage s+1 run under the arithmetic of stage s.
// * Prologue, once per element: d = softplus(dt * rstd + dt_bias) and d*x
//   (float2 per (token, channel)); B and C widened to float32 (and RMS-normed
//   per token when asked).
// * Recurrence: per token each lane updates its 4 states with packed f32x2
//   multiply/FMA and forms its partial C.h.  Every G tokens the G lanes of a
//   channel exchange partials in log2(G) shuffle rounds so that lane q ends
//   with the complete C.h of token q of the group (a transposing
//   reduction: G-1 shuffles per lane per G tokens) and applies the skip
//   term, the gate and the bf16 rounding for that one token.
// * exp(d A) costs one SFU ex2 per state; the SFU issues 16 per SM per
//   clock, a quarter of what the other work needs, so SWX of the 4 states
//   of a lane take a second exponential on the FMA pipe instead: Cody-Waite
//   reduction 2^x = 2^j 2^f with j = round(x), and a degree-5 polynomial
//   for 2^f on [-1/2, 1/2] (coefficients and their fit in
//   gen_exp2_poly.py; max relative error 1.9e-7 in float32), 2^j applied
//   through the exponent field.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma.h"

#include <type_traits>

namespace ssm {
namespace {

using namespace sm100;

constexpr int kTL = 32;  // tokens per stage
constexpr int kNS = 2;   // stages in flight
constexpr long long kWaitLimit = 2000000000ll;

// 1.5 * 2^23 + 127: adding it rounds x to an integer j held in the low
// mantissa bits, biased by 127 so that (bits << 23) is the float 2^j.
constexpr float kMagic = 12583039.0f;
constexpr float kP1 = 6.931468844e-01f, kP2 = 2.402223796e-01f, kP3 = 5.550893024e-02f,
                kP4 = 9.671698324e-03f, kP5 = 1.321867225e-03f;

// 2^(d*A2) for two states on the FMA pipe, for d >= 0 and A2 < 0 (a decay):
// d is first clamped to lim = -127 / A2 so that the exponent never drops below
// -127, where the result is exactly 0.
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
__device__ __forceinline__ float exp2_fma1(float d, float A2, float lim) {
  const float dc = fminf(d, lim);
  const float t = fmaf(dc, A2, kMagic);
  const float r = t - kMagic;
  const float f = fmaf(dc, A2, -r);
  float p = fmaf(kP5, f, kP4);
  p = fmaf(p, f, kP3);
  p = fmaf(p, f, kP2);
  p = fmaf(p, f, kP1);
  p = fmaf(p, f, 1.f);
  return p * __uint_as_float(__float_as_uint(t) << 23);
}

// Lane q of a group of G lanes holds partials p[u] of tokens u = 0..G-1; on
// return it holds the sum over the group of token q's partials.
template <int G>
__device__ __forceinline__ float transpose_reduce(float (&p)[G], int q) {
#pragma unroll
  for (int o = G / 2; o >= 1; o >>= 1) {
    const bool up = q & o;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? p[i] : p[i + o];
      const float keep = up ? p[i + o] : p[i];
      p[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return p[0];
}

template <int N, typename T, int CT>
struct alignas(128) M1Smem {
  T x[kNS][kTL][CT];
  T dt[kNS][kTL][CT];
  T z[kNS][kTL][CT];
  T B[kNS][kTL][N];
  T C[kNS][kTL][N];
  float2 ddx[kTL][CT];      // (d, d*x)
  float bc[kTL][2][N];      // B, C in float32
  T y[kTL][CT];
  uint64_t full[kNS];
};

// SPL states per lane (2 or 4), G = N / SPL lanes per channel.  SWX of a
// lane's SPL decays use the FMA-pipe exp2.  STATES: also store every token's
// state.
// PK: packed f32x2 state arithmetic (else scalar); UT: token groups per loop
// iteration (2 lets one group's shuffle reduction overlap the next group's
// arithmetic).
template <int N, typename T, int CT, bool HAS_Z, int SWX, int SPL, bool STATES, bool PK, int UT,
          bool WR = false>
__global__ void __launch_bounds__(CT *(N / SPL))
    m1_scan_tma_kernel(const __grid_constant__ CUtensorMap mx,
                       const __grid_constant__ CUtensorMap mdt,
                       const __grid_constant__ CUtensorMap mz,
                       const __grid_constant__ CUtensorMap mB,
                       const __grid_constant__ CUtensorMap mC, const M1Params p) {
  constexpr int G = N / SPL;  // lanes per channel
  constexpr int NT = CT * G;
  constexpr int NP = SPL / 2;  // state pairs per lane
  constexpr bool kBF16 = sizeof(T) == 2;
  static_assert(!WR || PK, "the state write is carried by the packed form only");
  using S = M1Smem<N, T, CT>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  S &s = *reinterpret_cast<S *>(smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u));

  const int64_t L = p.L, C = p.C, Gr = p.G;
  const int b = blockIdx.y;
  const int64_t c0 = (int64_t)blockIdx.x * CT;
  const int tid = threadIdx.x;
  const int cl = tid / G, q = tid % G;
  const int64_t c = c0 + cl;
  const bool cvalid = c < C;
  const int g = (int)(c0 / (C / Gr));
  const int nst = (int)((L + kTL - 1) / kTL);
  const bool softplus_on = p.flags & 1u;
  const bool rms_bc = p.flags & 2u;
  constexpr uint32_t kStageBytes = (3 * kTL * CT + 2 * kTL * N) * sizeof(T);
  constexpr uint32_t kStageBytesNoZ = (2 * kTL * CT + 2 * kTL * N) * sizeof(T);

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) mbar_init(&s.full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int stage) {
    const int buf = stage % kNS, t0 = stage * kTL;
    mbar_expect_tx(&s.full[buf], HAS_Z ? kStageBytes : kStageBytesNoZ);
    tma_load_3d(&s.x[buf][0][0], &mx, &s.full[buf], (int)c0, t0, b);
    tma_load_3d(&s.dt[buf][0][0], &mdt, &s.full[buf], (int)c0, t0, b);
    if (HAS_Z) tma_load_3d(&s.z[buf][0][0], &mz, &s.full[buf], (int)c0, t0, b);
    tma_load_3d(&s.B[buf][0][0], &mB, &s.full[buf], g * N, t0, b);
    tma_load_3d(&s.C[buf][0][0], &mC, &s.full[buf], g * N, t0, b);
  };
  if (tid == 0)
    for (int i = 0; i < kNS && i < nst; ++i) issue(i);

  float h[SPL], A2[SPL], lim[SPL];
#pragma unroll
  for (int j = 0; j < SPL; ++j) {
    h[j] = (cvalid && p.h0) ? p.h0[(b * C + c) * N + SPL * q + j] : 0.f;
    A2[j] = cvalid ? p.A[c * N + SPL * q + j] * kLog2e : 0.f;
    lim[j] = A2[j] < 0.f ? -127.f / A2[j] : 3.0e38f;
  }
  // The FMA-pipe exponential assumes decays (d >= 0, A < 0); a warp where any
  // of its states could grow uses the SFU for all of them.
  bool sw_ok = softplus_on;
#pragma unroll
  for (int j = SPL - SWX; j < SPL; ++j) sw_ok = sw_ok && (A2[j] < 0.f || !cvalid);
  sw_ok = __all_sync(0xffffffffu, sw_ok);
  const float Dc = (cvalid && p.D) ? p.D[c] : 0.f;
  // Prologue mapping: this thread always handles column pc of the tile.
  constexpr int TPR = NT / CT;
  const int pc = tid % CT, pt0 = tid / CT;
  const bool pvalid = c0 + pc < C;
  const float bias_pc = (pvalid && p.dt_bias) ? p.dt_bias[c0 + pc] : 0.f;

  for (int sg = 0; sg < nst; ++sg) {
    const int buf = sg % kNS;
    const int64_t t0 = (int64_t)sg * kTL;
    const int tn = (int)(L - t0 < kTL ? L - t0 : kTL);
    const bool ok = mbar_wait(&s.full[buf], (sg / kNS) & 1, kWaitLimit);
    if (__syncthreads_or(!ok)) {
      if (tid == 0 && p.status) atomicExch(p.status, 1);
      return;
    }
    // ---- prologue, once per (token, channel) and per (token, B/C row)
#pragma unroll 4
    for (int t = pt0; t < kTL; t += TPR) {
      float dv = 0.f, xv = 0.f;
      if (t < tn && pvalid) {
        xv = ld(&s.x[buf][t][pc]);
        dv = ld(&s.dt[buf][t][pc]);
        if (p.rstd) dv *= p.rstd[b * L + t0 + t];
        dv += bias_pc;
        if (softplus_on) dv = softplus_sfu(dv);
      }
      s.ddx[t][pc] = make_float2(dv, dv * xv);
    }
    for (int e = tid; e < kTL * 2; e += NT) {
      const int t = e >> 1, which = e & 1;
      const T *src = which ? s.C[buf][t] : s.B[buf][t];
      float v[N];
      float ss = 0.f;
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int n = 0; n < N; n += 8) {
          const uint4 w = *reinterpret_cast<const uint4 *>(src + n);
          v[n] = bf16lo(w.x); v[n + 1] = bf16hi(w.x); v[n + 2] = bf16lo(w.y); v[n + 3] = bf16hi(w.y);
          v[n + 4] = bf16lo(w.z); v[n + 5] = bf16hi(w.z); v[n + 6] = bf16lo(w.w); v[n + 7] = bf16hi(w.w);
        }
      } else {
#pragma unroll
        for (int n = 0; n < N; n += 4) {
          const float4 w = *reinterpret_cast<const float4 *>(src + n);
          v[n] = w.x; v[n + 1] = w.y; v[n + 2] = w.z; v[n + 3] = w.w;
        }
      }
#pragma unroll
      for (int n = 0; n < N; ++n) {
        if (t >= tn) v[n] = 0.f;
        ss += v[n] * v[n];
      }
      const float r = rms_bc ? rsqrtf(ss / N + p.eps) : 1.f;
#pragma unroll
      for (int n = 0; n < N; n += 4)
        *reinterpret_cast<float4 *>(&s.bc[t][which][n]) =
            make_float4(v[n] * r, v[n + 1] * r, v[n + 2] * r, v[n + 3] * r);
    }
    __syncthreads();

    // ---- recurrence, G tokens at a time, UT groups per iteration.  With a
    // state write, only the group holding the written token takes the form
    // that lets y read the written state; the others run the plain body.
    const int tw = (WR && p.t_write >= t0 && p.t_write < t0 + tn) ? (int)(p.t_write - t0) : -1;
#pragma unroll 1
    for (int tg0 = 0; tg0 < kTL; tg0 += G * UT) {
      auto group = [&](auto wr) {
#pragma unroll
        for (int ug = 0; ug < UT; ++ug) {
          const int tg = tg0 + ug * G;
          float part[G];
#pragma unroll
          for (int u = 0; u < G; ++u) {
            const int t = tg + u;
            const float2 ddx = s.ddx[t][cl];
            const float d = ddx.x, dx = ddx.y;
            float bv[SPL], cv[SPL], a[SPL];
            if constexpr (SPL >= 4) {
#pragma unroll
              for (int v = 0; v < SPL / 4; ++v) {
                const float4 b4 = *reinterpret_cast<const float4 *>(&s.bc[t][0][SPL * q + 4 * v]);
                const float4 c4 = *reinterpret_cast<const float4 *>(&s.bc[t][1][SPL * q + 4 * v]);
                bv[4 * v] = b4.x; bv[4 * v + 1] = b4.y; bv[4 * v + 2] = b4.z; bv[4 * v + 3] = b4.w;
                cv[4 * v] = c4.x; cv[4 * v + 1] = c4.y; cv[4 * v + 2] = c4.z; cv[4 * v + 3] = c4.w;
              }
            } else {
              const float2 b2 = *reinterpret_cast<const float2 *>(&s.bc[t][0][2 * q]);
              const float2 c2 = *reinterpret_cast<const float2 *>(&s.bc[t][1][2 * q]);
              bv[0] = b2.x; bv[1] = b2.y;
              cv[0] = c2.x; cv[1] = c2.y;
            }
            if constexpr (PK) {
#pragma unroll
              for (int pr = 0; pr < NP; ++pr) {
                const bool fma_pair = (SWX == 2 && SPL == 4 && pr == 1) && sw_ok;
                const bool fma_last = (SWX == 1 && pr == NP - 1) && sw_ok;
                if (fma_pair) {
                  const f2 e = exp2_fma2(d, mk2(A2[2], A2[3]), mk2(lim[2], lim[3]));
                  a[2] = e.x; a[3] = e.y;
                } else {
                  const f2 xx = mul2(mk2(d, d), mk2(A2[2 * pr], A2[2 * pr + 1]));
                  a[2 * pr] = ex2(xx.x);
                  a[2 * pr + 1] =
                      fma_last ? exp2_fma1(d, A2[2 * pr + 1], lim[2 * pr + 1]) : ex2(xx.y);
                }
              }
              const f2 dx2 = mk2(dx, dx);
              f2 yacc = mk2(0.f, 0.f);
              if constexpr (decltype(wr)::value) {
                // a state written at this token replaces h_t before y_t reads
                // it ("Mamba", nnterp guide, "The state")
#pragma unroll
                for (int pr = 0; pr < NP; ++pr) {
                  const f2 hn = fma2(mk2(a[2 * pr], a[2 * pr + 1]), mk2(h[2 * pr], h[2 * pr + 1]),
                                     mul2(dx2, mk2(bv[2 * pr], bv[2 * pr + 1])));
                  h[2 * pr] = hn.x;
                  h[2 * pr + 1] = hn.y;
                }
                if (t == tw && cvalid) {
#pragma unroll
                  for (int j = 0; j < SPL; ++j) h[j] = p.state_write[(b * C + c) * N + SPL * q + j];
                }
#pragma unroll
                for (int pr = 0; pr < NP; ++pr)
                  yacc = fma2(mk2(cv[2 * pr], cv[2 * pr + 1]), mk2(h[2 * pr], h[2 * pr + 1]), yacc);
              } else {
#pragma unroll
                for (int pr = 0; pr < NP; ++pr) {
                  const f2 hn = fma2(mk2(a[2 * pr], a[2 * pr + 1]), mk2(h[2 * pr], h[2 * pr + 1]),
                                     mul2(dx2, mk2(bv[2 * pr], bv[2 * pr + 1])));
                  h[2 * pr] = hn.x;
                  h[2 * pr + 1] = hn.y;
                  yacc = fma2(mk2(cv[2 * pr], cv[2 * pr + 1]), hn, yacc);
                }
              }
              part[u] = yacc.x + yacc.y;
            } else {
#pragma unroll
              for (int j = 0; j < SPL; ++j) {
                const bool fma_j = (j >= SPL - SWX) && sw_ok;
                a[j] = fma_j ? exp2_fma1(d, A2[j], lim[j]) : ex2(d * A2[j]);
              }
              float acc = 0.f;
#pragma unroll
              for (int j = 0; j < SPL; ++j) {
                h[j] = fmaf(a[j], h[j], dx * bv[j]);
                acc = fmaf(cv[j], h[j], acc);
              }
              part[u] = acc;
            }
            if constexpr (STATES) {
              if (cvalid && t < tn) {
                float *sp = p.states + ((b * L + t0 + t) * C + c) * N + SPL * q;
#pragma unroll
                for (int j = 0; j < SPL; j += 2)
                  *reinterpret_cast<float2 *>(sp + j) = make_float2(h[j], h[j + 1]);
              }
            }
          }
          const float yq = transpose_reduce<G>(part, q);
          const int tt = tg + q;  // this lane's token
          if (tt < tn && cvalid) {
            float yv = yq + Dc * ld(&s.x[buf][tt][cl]);
            if (HAS_Z) {
              const float zv = ld(&s.z[buf][tt][cl]);
              yv *= kBF16 ? silu_tanh(zv) : silu(zv);
            }
            st(&s.y[tt][cl], yv);
          }
        }
      };
      if constexpr (WR) {
        if (tw >= tg0 && tw < tg0 + G * UT)
          group(std::true_type{});
        else
          group(std::false_type{});
      } else {
        group(std::false_type{});
      }
    }
    __syncthreads();
    // ---- next loads into this buffer, then the y tile
    if (tid == 0 && sg + kNS < nst) issue(sg + kNS);
    {
      constexpr int kChunk = 16 / sizeof(T);   // elements per 16-byte store
      constexpr int kPerRow = CT / kChunk;
      T *y = static_cast<T *>(p.y);
      for (int e = tid; e < tn * kPerRow; e += NT) {
        const int t = e / kPerRow, k = e % kPerRow;
        const int64_t cg = c0 + k * kChunk;
        T *dst = y + (b * L + t0 + t) * C + cg;
        if (cg + kChunk <= C) {
          *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(&s.y[t][k * kChunk]);
        } else {
          for (int i = 0; i < kChunk && cg + i < C; ++i) dst[i] = s.y[t][k * kChunk + i];
        }
      }
    }
  }
  if (p.h_last && cvalid) {
    float *hp = p.h_last + (b * C + c) * N + SPL * q;
#pragma unroll
    for (int j = 0; j < SPL; j += 2) *reinterpret_cast<float2 *>(hp + j) = make_float2(h[j], h[j + 1]);
  }
}

template <typename T>
CUtensorMapDataType tmap_type() {
  return sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
}

template <int N, typename T, int CT, bool HZ, int SWX, int SPL, bool ST, bool PK = true,
          int UT = 1, bool WR = false>
cudaError_t launch_tma(const M1Params &p, cudaStream_t s) {
  CUtensorMap mx, mdt, mz, mB, mC;
  const uint64_t es = sizeof(T);
  {
    uint64_t dims[3] = {(uint64_t)p.C, (uint64_t)p.L, (uint64_t)p.batch};
    uint64_t strides[2] = {(uint64_t)p.C * es, (uint64_t)(p.L * p.C) * es};
    uint32_t box[3] = {(uint32_t)CT, (uint32_t)kTL, 1};
    if (!encode_tiled(&mx, tmap_type<T>(), 3, p.x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tiled(&mdt, tmap_type<T>(), 3, p.dt, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    if (HZ && !encode_tiled(&mz, tmap_type<T>(), 3, p.z, dims, strides, box,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    if (!HZ) mz = mx;
  }
  {
    const uint64_t GN = (uint64_t)(p.G * p.N);
    uint64_t dims[3] = {GN, (uint64_t)p.L, (uint64_t)p.batch};
    uint64_t strides[2] = {GN * es, (uint64_t)p.L * GN * es};
    uint32_t box[3] = {(uint32_t)N, (uint32_t)kTL, 1};
    if (!encode_tiled(&mB, tmap_type<T>(), 3, p.B, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tiled(&mC, tmap_type<T>(), 3, p.Cm, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  auto k = m1_scan_tma_kernel<N, T, CT, HZ, SWX, SPL, ST, PK, UT, WR>;
  const size_t smem = sizeof(M1Smem<N, T, CT>) + 128;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((unsigned)((p.C + CT - 1) / CT), (unsigned)p.batch);
  k<<<grid, CT * (N / SPL), smem, s>>>(mx, mdt, mz, mB, mC, p);
  return cudaGetLastError();
}

// Variant choice: per-token states (tests only) take one fixed form; the
// others follow p.variant (states per lane, packed math, unrolling, and 8 =
// one decay per lane on the FMA-pipe exp2).
template <int N, typename T, bool HZ>
cudaError_t launch_v(const M1Params &p, cudaStream_t s) {
  if (p.states) return launch_tma<N, T, 16, HZ, 0, 4, true>(p, s);
  // a state written at one token: the default lane split, with the write
  if (p.state_write) return launch_tma<N, T, 16, HZ, 0, 2, false, true, 1, true>(p, s);
  // variant = 4 * (packed) + 2 * (two groups per iteration) + (2 states per lane)
  const bool ok32 = p.G == 1 || (p.C / p.G) % 32 == 0;
  switch (p.variant) {
    case 0: return launch_tma<N, T, 16, HZ, 0, 4, false, false, 1>(p, s);
    case 1: return launch_tma<N, T, 16, HZ, 0, 2, false, false, 1>(p, s);
    case 2: return launch_tma<N, T, 16, HZ, 0, 4, false, false, 2>(p, s);
    case 3: return launch_tma<N, T, 16, HZ, 0, 2, false, false, 2>(p, s);
    case 4: return launch_tma<N, T, 16, HZ, 0, 4, false, true, 1>(p, s);
    case 5: return launch_tma<N, T, 16, HZ, 0, 2, false, true, 1>(p, s);
    case 6: return launch_tma<N, T, 16, HZ, 0, 4, false, true, 2>(p, s);
    case 7: return launch_tma<N, T, 16, HZ, 0, 2, false, true, 2>(p, s);
    case 8: return launch_tma<N, T, 16, HZ, 1, 4, false, true, 1>(p, s);
    // 9..12: 32-channel tiles (a tile must not straddle two B/C groups,
    // else the default form runs)
    case 9:
      if (ok32) return launch_tma<N, T, 32, HZ, 0, 4, false, true, 1>(p, s);
      break;
    case 10:
      if (ok32) return launch_tma<N, T, 32, HZ, 0, 8, false, true, 1>(p, s);
      break;
    case 11:
      if (ok32) return launch_tma<N, T, 32, HZ, 0, 2, false, true, 1>(p, s);
      break;
    case 12:
      if (ok32) return launch_tma<N, T, 32, HZ, 1, 4, false, true, 1>(p, s);
      break;
    case 13: return launch_tma<N, T, 16, HZ, 1, 2, false, true, 1>(p, s);
    case 14: return launch_tma<N, T, 16, HZ, 1, 2, false, true, 2>(p, s);
  }
  return launch_tma<N, T, 16, HZ, 0, 2, false, true, 1>(p, s);
}

template <typename T>
cudaError_t launch_tma_t(const M1Params &p, cudaStream_t s) {
  const bool hz = p.z != nullptr;
  switch (p.N) {
    case 8: return hz ? launch_tma<8, T, 16, true, 0, 4, false>(p, s)
                      : launch_tma<8, T, 16, false, 0, 4, false>(p, s);
    case 16: return hz ? launch_v<16, T, true>(p, s) : launch_v<16, T, false>(p, s);
    case 32: return hz ? launch_tma<32, T, 16, true, 0, 4, false>(p, s)
                       : launch_tma<32, T, 16, false, 0, 4, false>(p, s);
  }
  return cudaErrorNotSupported;
}

}  // namespace

// The pipelined kernel needs 16-byte rows for TMA (a 16-channel tile and the
// B/C rows), a channel tile inside one group, and N in {8, 16, 32}; per-token
// states only with N = 16.
bool m1_scan_tma_supported(const M1Params &p) {
  if (p.states && p.N != 16) return false;
  const int64_t es = p.io == 1 ? 2 : 4;
  if (p.N != 8 && p.N != 16 && p.N != 32) return false;
  if ((p.N * es) % 16 || (p.C * es) % 16 || (p.G * p.N * es) % 16) return false;
  if (p.G > 1 && (p.C / p.G) % 16) return false;
  if (p.L >= (1ll << 31) || p.C >= (1ll << 31) || p.batch > 65535) return false;
  return true;
}

cudaError_t launch_m1_scan_tma(const M1Params &p, cudaStream_t s) {
  return p.io == 1 ? launch_tma_t<__nv_bfloat16>(p, s) : launch_tma_t<float>(p, s);
}

}  // namespace ssm
