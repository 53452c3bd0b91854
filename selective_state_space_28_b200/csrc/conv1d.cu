// conv1d.cu -- causal depthwise convolution over tokens, then silu: the
// mixers' conv1d ("Mamba-2", nnterp encyclopedia: the module tree's
// Conv1d(channels, channels, kernel 4, padding 3, groups = channels) and "The
// mixer's values", x, B, C = silu(conv1d(xBC)); "Mamba", tokentrails, "Code":
// x = silu(causal_conv1d(x)), depthwise, width 4):
//
//   u[t, c] = silu(bias[c] + sum_{k<W} w[c, k] * x[t - (W - 1) + k, c]),
//
// inputs before t = 0 taken from the conv state (the W - 1 inputs before the
// sequence, oldest first; zeros without one); the state after the call is the
// last W - 1 inputs.  With seqlen 1 and the state updated in place this is the
// decode form of the same convolution.
//
// HBM-streaming layout: a thread owns V consecutive channels -- 8 bf16 (a
// 16-byte vector of the tokens-first rows) when the channel count is a
// multiple of 8, else 4 (8 bytes bf16, 16 bytes float32) -- over a run of
// tokens, keeps the W - 1 previous inputs in registers, and reads each input
// once (plus a W - 1 token halo at the start of its run, mostly from L2) and
// writes each output once; a warp covers 32 consecutive vectors of a row, so
// every access is coalesced.  The inputs reach the thread through its own
// shared-memory slots, copied asynchronously several batches ahead, so that
// enough bytes are in flight per SM without holding them in registers.  The
// arithmetic runs on channel pairs in packed f32x2.
#include "common.cuh"
#include "internal.h"

namespace ssm {
namespace {

constexpr int kRun = 128;  // tokens per thread (when the state is not updated in place)

// Streaming (evict-first) vector loads and stores through the compiler's
// intrinsics (the halo loads and the output stores).
// V channels a thread: 8 bf16 (16 bytes) where the channel count allows,
// else 4 (8 bytes); float32 takes 4 (16 bytes).
template <typename T, int V> struct Vec;
template <> struct Vec<__nv_bfloat16, 8> {
  static constexpr int V = 8;
  using Raw = uint4;
  static __device__ __forceinline__ Raw load(const __nv_bfloat16 *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
  }
  static __device__ __forceinline__ void widen(const Raw &w, float (&f)[8]) {
    f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
    f[4] = bf16lo(w.z); f[5] = bf16hi(w.z); f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&f)[8]) {
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                     pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
  }
};
template <> struct Vec<__nv_bfloat16, 4> {
  static constexpr int V = 4;
  using Raw = uint2;
  static __device__ __forceinline__ Raw load(const __nv_bfloat16 *p) {
    return __ldcs(reinterpret_cast<const uint2 *>(p));
  }
  static __device__ __forceinline__ void widen(const Raw &w, float (&f)[4]) {
    f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&f)[4]) {
    __stcs(reinterpret_cast<uint2 *>(p), make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3])));
  }
};
template <> struct Vec<float, 4> {
  static constexpr int V = 4;
  using Raw = float4;
  static __device__ __forceinline__ Raw load(const float *p) {
    return __ldcs(reinterpret_cast<const float4 *>(p));
  }
  static __device__ __forceinline__ void widen(const Raw &v, float (&f)[4]) {
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  static __device__ __forceinline__ void store(float *p, const float (&f)[4]) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(f[0], f[1], f[2], f[3]));
  }
};

template <typename T> __device__ __forceinline__ float act(float v, bool on) {
  if (!on) return v;
  return sizeof(T) == 2 ? silu_tanh(v) : silu(v);
}

// Vector form: channels % V == 0.  Thread =
// (batch row, vector of V channels, run of kRun tokens).  A thread's next
// kTok-token batches are copied into its own shared-memory slots with
// cp.async, kStages - 1 batches ahead: the copies in flight hold no
// registers, and each thread waits only for its own copies (no barrier).
// Four stages of 8 tokens measured best for bf16 (24 tokens, 192 bytes in
// flight per thread); float32 vectors, twice the size, keep three.
constexpr int kTok = 8;
constexpr int kStages = 4;

template <int BYTES>
__device__ __forceinline__ void cp_async(void *dst, const void *src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(d), "l"(src), "n"(BYTES)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T, int W, int VW>
__global__ void __launch_bounds__(128)
    conv1d_vec_kernel(ConvParams p) {
  using VT = Vec<T, VW>;
  constexpr int V = VT::V;
  using Raw = typename VT::Raw;
  constexpr int NS = sizeof(Raw) == 16 ? 3 : kStages;
  constexpr int NT = sizeof(Raw) == 16 ? 8 : kTok;
  __shared__ Raw stage[NS][NT][128];
  const int64_t nvec = p.Cc / V;
  const int64_t gv = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gv >= nvec * p.batch) return;
  const int64_t b = gv / nvec, c0 = (gv % nvec) * V;
  const int64_t L = p.L, Cc = p.Cc;
  const int64_t t0 = (int64_t)blockIdx.y * p.run;
  if (t0 >= L) return;
  const int64_t t1 = t0 + p.run < L ? t0 + p.run : L;
  const T *x = static_cast<const T *>(p.x);
  T *u = static_cast<T *>(p.u);
  const int tid = threadIdx.x;
  const int nb = (int)((t1 - t0 + NT - 1) / NT);  // batches in this run

  const T *px = x + (b * L + t0) * Cc + c0;  // next row to copy
  int64_t tc = t0;                            // its token
  auto issue = [&](int slot) {
#pragma unroll
    for (int a = 0; a < NT; ++a) {
      if (tc < t1) cp_async<sizeof(Raw)>(&stage[slot][a][tid], px);
      px += Cc;
      ++tc;
    }
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < NS - 1; ++s) issue(s);

  // The arithmetic runs on channel pairs (packed f32x2: each lane of a pair
  // is exactly the scalar fmaf / multiply), half the instructions of
  // channel by channel; the bits are those of the scalar form and of the
  // fused scan's convolution.
  constexpr int VP = V / 2;
  f2 w[VP][W], bias[VP];
#pragma unroll
  for (int v = 0; v < VP; ++v) {
#pragma unroll
    for (int k = 0; k < W; ++k)
      w[v][k] = mk2(p.w[(c0 + 2 * v) * W + k], p.w[(c0 + 2 * v + 1) * W + k]);
    bias[v] = p.bias ? mk2(p.bias[c0 + 2 * v], p.bias[c0 + 2 * v + 1]) : mk2(0.f, 0.f);
  }
  // hist[j][v]: input j + 1 tokens before the current one (j < W - 1)
  f2 hist[W > 1 ? W - 1 : 1][VP];
#pragma unroll
  for (int j = 0; j < W - 1; ++j) {
    const int64_t tau = t0 - 1 - j;
    float hv[V];
    if (tau >= 0) {
      VT::widen(VT::load(x + (b * L + tau) * Cc + c0), hv);
    } else {
#pragma unroll
      for (int v = 0; v < V; ++v)
        hv[v] = p.state_in ? p.state_in[((b * Cc) + c0 + v) * (W - 1) + (W - 1) + tau] : 0.f;
    }
#pragma unroll
    for (int v = 0; v < VP; ++v) hist[j][v] = mk2(hv[2 * v], hv[2 * v + 1]);
  }
  const f2 half2 = mk2(0.5f, 0.5f);
  T *pu = u + (b * L + t0) * Cc + c0;
  for (int i = 0; i < nb; ++i) {
    issue((i + NS - 1) % NS);  // the slot batch i - 1 used (an empty group past the end)
    cp_async_wait<NS - 1>();   // batch i has landed
    const int slot = i % NS;
    const int na = (int)(t1 - (t0 + (int64_t)i * NT) < NT ? t1 - (t0 + (int64_t)i * NT) : NT);
#pragma unroll
    for (int a = 0; a < NT; ++a) {
      if (a >= na) break;
      float xs[V], o[V];
      VT::widen(stage[slot][a][tid], xs);
      f2 xv[VP];
#pragma unroll
      for (int v = 0; v < VP; ++v) xv[v] = mk2(xs[2 * v], xs[2 * v + 1]);
#pragma unroll
      for (int v = 0; v < VP; ++v) {
        f2 acc = fma2(w[v][W - 1], xv[v], bias[v]);
#pragma unroll
        for (int j = 0; j < W - 1; ++j) acc = fma2(w[v][W - 2 - j], hist[j][v], acc);
        if (sizeof(T) == 2 && p.silu) {
          // silu(z) = z (1 + tanh(z / 2)) / 2, as silu_tanh
          const f2 hz = mul2(half2, acc);
          float ta, tb;
          asm("tanh.approx.f32 %0, %1;" : "=f"(ta) : "f"(hz.x));
          asm("tanh.approx.f32 %0, %1;" : "=f"(tb) : "f"(hz.y));
          const f2 u = mul2(acc, fma2(half2, mk2(ta, tb), half2));
          o[2 * v] = u.x;
          o[2 * v + 1] = u.y;
        } else {
          o[2 * v] = act<T>(acc.x, p.silu);
          o[2 * v + 1] = act<T>(acc.y, p.silu);
        }
      }
      VT::store(pu, o);
      pu += Cc;
#pragma unroll
      for (int j = W - 2; j > 0; --j)
#pragma unroll
        for (int v = 0; v < VP; ++v) hist[j][v] = hist[j - 1][v];
      if (W > 1) {
#pragma unroll
        for (int v = 0; v < VP; ++v) hist[0][v] = xv[v];
      }
    }
  }
  cp_async_wait<0>();
  // The run that ends the sequence leaves the state: the last W - 1 inputs,
  // oldest first (from before the sequence when it is shorter than that).
  if (p.state_out && t1 == L) {
#pragma unroll
    for (int j = 0; j < W - 1; ++j)
#pragma unroll
      for (int v = 0; v < VP; ++v) {
        p.state_out[((b * Cc) + c0 + 2 * v) * (W - 1) + (W - 2 - j)] = hist[j][v].x;
        p.state_out[((b * Cc) + c0 + 2 * v + 1) * (W - 1) + (W - 2 - j)] = hist[j][v].y;
      }
  }
}

// Scalar form, for any channel count: thread = (batch row, channel, run).
template <typename T, int W>
__global__ void __launch_bounds__(128)
    conv1d_scalar_kernel(ConvParams p) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= p.Cc * p.batch) return;
  const int64_t b = g / p.Cc, c = g % p.Cc;
  const int64_t L = p.L, Cc = p.Cc;
  const int64_t t0 = (int64_t)blockIdx.y * p.run;
  if (t0 >= L) return;
  const int64_t t1 = t0 + p.run < L ? t0 + p.run : L;
  const T *x = static_cast<const T *>(p.x);
  T *u = static_cast<T *>(p.u);
  float w[W];
#pragma unroll
  for (int k = 0; k < W; ++k) w[k] = p.w[c * W + k];
  const float bias = p.bias ? p.bias[c] : 0.f;
  float hist[W > 1 ? W - 1 : 1];
#pragma unroll
  for (int j = 0; j < W - 1; ++j) {
    const int64_t tau = t0 - 1 - j;
    hist[j] = tau >= 0 ? ld(x + (b * L + tau) * Cc + c)
                       : (p.state_in ? p.state_in[(b * Cc + c) * (W - 1) + (W - 1) + tau] : 0.f);
  }
  for (int64_t t = t0; t < t1; ++t) {
    const float xv = ld(x + (b * L + t) * Cc + c);
    float acc = fmaf(w[W - 1], xv, bias);
#pragma unroll
    for (int j = 0; j < W - 1; ++j) acc = fmaf(w[W - 2 - j], hist[j], acc);
    st(u + (b * L + t) * Cc + c, act<T>(acc, p.silu));
#pragma unroll
    for (int j = W - 2; j > 0; --j) hist[j] = hist[j - 1];
    if (W > 1) hist[0] = xv;
  }
  if (p.state_out && t1 == L) {
#pragma unroll
    for (int j = 0; j < W - 1; ++j) p.state_out[(b * Cc + c) * (W - 1) + (W - 2 - j)] = hist[j];
  }
}

// The widest vector whose rows the channel count fills (row bases are then
// 16-byte aligned): 8 (bf16) or 4 channels a thread, or 0 for the
// per-channel form.
template <typename T>
int vec_width(const ConvParams &p) {
  if (sizeof(T) == 2 && p.Cc % 8 == 0) return 8;
  return p.Cc % 4 == 0 ? 4 : 0;
}

// CTAs of a vector form resident per SM (its registers and slots decide),
// read once per instance from the runtime's occupancy calculator.
template <typename T, int W, int VW>
int vec_ctas_per_sm() {
  static const int n = [] {
    int k = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&k, conv1d_vec_kernel<T, W, VW>, 128, 0) !=
            cudaSuccess ||
        k <= 0) {
      cudaGetLastError();
      return 0;
    }
    return k;
  }();
  return n;
}

template <typename T, int W, int VW>
cudaError_t launch_vec(const ConvParams &p, cudaStream_t s) {
  const int64_t runs = (p.L + p.run - 1) / p.run;
  const int64_t units = p.batch * (p.Cc / VW);
  dim3 grid((unsigned)((units + 127) / 128), (unsigned)runs);
  // the slots (32-48 KB per CTA) need the shared-memory carve-out for
  // several CTAs per SM (a preference of the current device: set per call)
  if (cudaFuncSetAttribute(conv1d_vec_kernel<T, W, VW>,
                           cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    cudaGetLastError();  // a preference only: never fail the call on it
  conv1d_vec_kernel<T, W, VW><<<grid, 128, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int W>
cudaError_t launch_w(const ConvParams &p, cudaStream_t s) {
  switch (vec_width<T>(p)) {
    case 8:
      if constexpr (sizeof(T) == 2) return launch_vec<T, W, 8>(p, s);
      break;
    case 4: return launch_vec<T, W, 4>(p, s);
  }
  const int64_t runs = (p.L + p.run - 1) / p.run;
  dim3 grid((unsigned)((p.batch * p.Cc + 127) / 128), (unsigned)runs);
  conv1d_scalar_kernel<T, W><<<grid, 128, 0, s>>>(p);
  return cudaGetLastError();
}

// Tokens per thread of a vector form: whole batches of kTok, at least
// kRunMin, chosen so that the grid fills whole waves of resident CTAs.  With
// kRun tokens the bf16 2.7B mixer (b4, 5376 channels, 8 a thread: 21 x 32
// CTAs) would leave the last wave part empty; runs fitted to the resident
// CTAs fill it.
constexpr int64_t kRunMin = 64;
template <typename T, int W, int VW>
int64_t fitted_run(const ConvParams &p) {
  const int64_t bx = (p.batch * (p.Cc / VW) + 127) / 128;
  const int64_t per_sm = vec_ctas_per_sm<T, W, VW>();
  if (per_sm <= 0 || bx <= 0) return kRun;
  const int64_t cap = (int64_t)device_sm_count() * per_sm;
  const int64_t runs0 = (p.L + kRun - 1) / kRun;
  int64_t waves = bx * runs0 / cap;  // whole waves the default runs fill
  if (waves < 1) waves = 1;
  int64_t runs = cap * waves / bx;  // runs of each column that fit in them
  if (runs < 1) runs = 1;
  int64_t run = (p.L + runs - 1) / runs;
  run = (run + kTok - 1) / kTok * kTok;
  return run < kRunMin ? kRunMin : run;
}

template <typename T, int W>
int64_t run_w(const ConvParams &p) {
  switch (vec_width<T>(p)) {
    case 8:
      if constexpr (sizeof(T) == 2) return fitted_run<T, W, 8>(p);
      break;
    case 4: return fitted_run<T, W, 4>(p);
  }
  return kRun;
}

template <typename T>
cudaError_t launch_t(const ConvParams &p, cudaStream_t s) {
  switch (p.W) {
    case 1: return launch_w<T, 1>(p, s);
    case 2: return launch_w<T, 2>(p, s);
    case 3: return launch_w<T, 3>(p, s);
    case 4: return launch_w<T, 4>(p, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
int64_t run_t(const ConvParams &p) {
  switch (p.W) {
    case 1: return run_w<T, 1>(p);
    case 2: return run_w<T, 2>(p);
    case 3: return run_w<T, 3>(p);
    case 4: return run_w<T, 4>(p);
  }
  return kRun;
}

}  // namespace

// Tokens per thread: the whole sequence when the state is updated in place
// (the run that reads the incoming state must be the one that writes the new
// state), else a run fitted to the device's waves (vector form) or kRun.
int64_t conv1d_run_length(const ConvParams &p, bool state_in_place) {
  if (state_in_place) return p.L > 0 ? p.L : 1;
  return p.io == 1 ? run_t<__nv_bfloat16>(p) : run_t<float>(p);
}

bool conv1d_supported(const ConvParams &p) {
  const int64_t run = p.run > 0 ? p.run : 1;
  return p.W >= 1 && p.W <= kConvMaxWidth && (p.L + run - 1) / run <= 65535 &&
         (p.batch * p.Cc + 127) / 128 < (1ll << 31);
}

cudaError_t launch_conv1d(const ConvParams &p, cudaStream_t s) {
  return p.io == 1 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace ssm
