// scan_m1_tma.cu -- Mamba-1 selective scan, pipelined form (kernel a).
//
// Same arithmetic as scan_m1.cu ("Mamba", nnterp guide, intro and "The
// values"; "Mamba", tokentrails, "Code"; "Falcon-Mamba", "Where the norms
// sit"):
//   d = softplus(dt * rstd + dt_bias[c]);  h[n] = exp(d A[c,n]) h[n] + d B[n] x
//   y = C . h + D[c] x;  y *= silu(z)
// organised for throughput on sm_100a.
//
// Work split.  A CTA owns one batch row, 32 channels and one segment of the
// sequence.  Each channel's N states sit in G = N/4 lanes of one warp, four
// float32 states per lane, in registers; a warp holds 32/G channels.  The
// segment is walked in stages of 32 tokens that TMA brings into a ring of NS
// stage buffers (x, dt, z as [32 tokens x 32 channels], B and C as
// [32 tokens x N]).
//
// Per stage, every warp (no CTA-wide barrier anywhere in the loop):
//   1. waits for the stage's bytes (mbarrier `full`);
//   2. for its share of the stage's tokens and all 32 channels computes
//      d = softplus(dt rstd + bias), d x, D x and silu(z) (with
//      SSM_RMSNORM_BC also each token's 1/rms of B_t, folded into d x, and
//      of C_t, kept for the readout), then arrives on `conv`;
//   3. waits on `conv` (every warp's share), then runs the recurrence, B and
//      C read as they landed: per token each lane updates its four states
//      with packed f32x2 arithmetic and forms its partial C.h, the decays of
//      the next 8 tokens formed while the current 8 run their chain; every G
//      tokens the G lanes of a channel trade partials in log2(G) shuffle
//      rounds so that lane q ends with token q's complete C.h (a transposing
//      reduction), and applies C_t's factor, the skip term, the gate and the
//      rounding for that token;
//   4. arrives on `empty` (the issuing thread refills a stage's buffer once
//      every warp has released it) and stores its rows of the previous
//      stage's y, which every warp has finished by now, in whole 64-byte
//      rows.
//
// Sequence segments (the carry across chunks).  When batch x channels gives
// too few warps to fill the SMs, the sequence is cut into S segments and run
// in three launches: (1) segments 0..S-2 scanned from their own start (h0 for
// the first, zeros for the others) without any readout, leaving their end
// states and the sum of their steps; (2) a carry kernel that chains them: the
// state entering segment k+1 is P_k * (state entering k) + E_k with
// P_k[n] = exp(A[c,n] * sum of the segment's steps), evaluated as an
// inclusive warp-shuffle scan over the (P, E) pairs, which compose
// associatively; (3) every segment rescanned from its entering state with the
// readout.  Rescanning from the carried state computes exactly
// h_t = (local state from zero)_t + (prod of decays)_t * carry, the fix-up,
// without storing the local states.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma.h"

#include <algorithm>
#include <type_traits>
#include <cmath>

namespace ssm {
namespace {

using namespace sm100;

constexpr int kTL = 32;  // tokens per stage
constexpr int kCT = 32;  // channels per CTA
constexpr long long kWaitLimit = 2000000000ll;  // clock cycles (about one second)

enum { kModeFull = 0, kModeStateOnly = 1 };

// Decays per lane (of 4) taken by the FMA-pipe exp2 instead of the SFU (0 or
// 2): the SFU issues 16 exponentials per SM per clock, the FMA pipe 128
// lane-operations, so moving a share of the decays balances the two.
constexpr int kPolyStates = 0;

template <int N, typename T, int NS>
struct alignas(128) ScanSmem {
  T x[NS][kTL][kCT];
  T dt[NS][kTL][kCT];
  T z[NS][kTL][kCT];
  T B[NS][kTL][N];
  T C[NS][kTL][N];
  // Per (token, channel) of a stage: (d, d*x) for the recurrence and
  // (D*x, silu(z)) for the epilogue.  Two buffers by stage parity: a warp
  // that has finished stage s writes stage s+1's values while another still
  // reads stage s's (no warp gets further ahead: the next stage's scan waits
  // for every warp's `conv` arrival).  Rows are padded by 16 bytes so that a
  // warp's lanes, one row each, fall in distinct banks.
  float2 ddx[2][kTL][kCT + 2];
  float2 eg[2][kTL][kCT + 2];
  // With RMS norms on B and C: each token's factor 1 / rms(C_t), by stage
  // parity like eg (the factor of B_t is folded into d * x).
  float rc[2][kTL];
  // Output staging, two buffers by stage parity: the warps write stage s's y
  // here, and during stage s+1 (once the `conv` barrier shows every warp has
  // finished stage s) each warp stores a quarter of its rows to global
  // memory in full 32-channel rows -- whole 32-byte sectors, so that HBM3e
  // (no write mask) never has to merge a partly written sector.
  T y[2][kTL][kCT];
  float bias[kCT], skip[kCT];
  uint64_t full[NS], conv[NS], empty[NS], ylast;
};

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

// J consecutive I/O values from shared memory, widened to float32 (bf16 -> f32
// is exact: the bf16 bits are the top half of the f32 bits).
template <int J, typename T>
__device__ __forceinline__ void widen(const T *src, float (&v)[J]) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (J == 8) {
      const uint4 w = *reinterpret_cast<const uint4 *>(src);
      v[0] = bf16lo(w.x); v[1] = bf16hi(w.x); v[2] = bf16lo(w.y); v[3] = bf16hi(w.y);
      v[4] = bf16lo(w.z); v[5] = bf16hi(w.z); v[6] = bf16lo(w.w); v[7] = bf16hi(w.w);
    } else if constexpr (J == 4) {
      const uint2 w = *reinterpret_cast<const uint2 *>(src);
      v[0] = bf16lo(w.x); v[1] = bf16hi(w.x); v[2] = bf16lo(w.y); v[3] = bf16hi(w.y);
    } else if constexpr (J == 2) {
      const uint32_t w = *reinterpret_cast<const uint32_t *>(src);
      v[0] = bf16lo(w); v[1] = bf16hi(w);
    } else {
      static_assert(J == 1, "1, 2, 4 or 8 values");
      v[0] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(src));
    }
  } else if constexpr (J == 1) {
    v[0] = *reinterpret_cast<const float *>(src);
  } else if constexpr (J % 4 == 0) {
#pragma unroll
    for (int i = 0; i < J; i += 4) {
      const float4 a = *reinterpret_cast<const float4 *>(src + i);
      v[i] = a.x; v[i + 1] = a.y; v[i + 2] = a.z; v[i + 3] = a.w;
    }
  } else {
    static_assert(J == 2, "2 or a multiple of 4 values");
    const float2 a = *reinterpret_cast<const float2 *>(src);
    v[0] = a.x; v[1] = a.y;
  }
}

// NP pairs of float32 (SPL = 2 NP consecutive values) from / to memory.
template <int NP>
__device__ __forceinline__ void load_pairs(const float *src, f2 (&v)[NP]) {
  if constexpr (NP == 2) {
    const float4 a = *reinterpret_cast<const float4 *>(src);
    v[0] = mk2(a.x, a.y);
    v[1] = mk2(a.z, a.w);
  } else {
    static_assert(NP == 1, "2 or 4 states per lane");
    const float2 a = *reinterpret_cast<const float2 *>(src);
    v[0] = mk2(a.x, a.y);
  }
}
// The same from a row of the I/O type: bfloat16 widens exactly to float32,
// so these are the values the widened copy would hold.
template <int NP, typename T>
__device__ __forceinline__ void load_pairs_io(const T *src, f2 (&v)[NP]) {
  if constexpr (sizeof(T) == 4) {
    load_pairs<NP>(reinterpret_cast<const float *>(src), v);
  } else if constexpr (NP == 2) {
    const uint2 a = *reinterpret_cast<const uint2 *>(src);
    v[0] = mk2(bf16lo(a.x), bf16hi(a.x));
    v[1] = mk2(bf16lo(a.y), bf16hi(a.y));
  } else {
    const uint32_t a = *reinterpret_cast<const uint32_t *>(src);
    v[0] = mk2(bf16lo(a), bf16hi(a));
  }
}
template <int NP>
__device__ __forceinline__ void store_pairs(float *dst, const f2 (&v)[NP]) {
  if constexpr (NP == 2)
    *reinterpret_cast<float4 *>(dst) = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
  else
    *reinterpret_cast<float2 *>(dst) = make_float2(v[0].x, v[0].y);
}

// MODE: full scan with readout, or state-only (segments' end states).
// STATES: also store every token's state.  A state written at a token
// (p.state_write) runs the full scan in three parts (see below).
// SPL: states per lane (4, or 2 for twice the warps on small problems).
template <int N, int SPL, typename T, int NS, bool HAS_Z, int MODE, bool STATES, int PX, bool RBC>
__global__ void __launch_bounds__(kCT *(N / SPL), N >= 32 ? 2 : 3)
    m1_scan_tma_kernel(const __grid_constant__ CUtensorMap mx,
                       const __grid_constant__ CUtensorMap mdt,
                       const __grid_constant__ CUtensorMap mz,
                       const __grid_constant__ CUtensorMap mB,
                       const __grid_constant__ CUtensorMap mC, const M1Params p) {
  constexpr int G = N / SPL;        // lanes per channel
  constexpr int NP = SPL / 2;       // state pairs per lane
  constexpr int CPW = 32 / G;       // channels per warp
  constexpr int NW = kCT / CPW;     // warps per CTA
  constexpr int TPW = kTL / NW;     // tokens each warp prepares per stage
  constexpr bool kBF16 = sizeof(T) == 2;
  constexpr bool kFull = MODE == kModeFull;
  static_assert(N % 8 == 0 || !kBF16, "bf16 rows of B and C are 16-byte multiples");
  using S = ScanSmem<N, T, NS>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  S &s = *reinterpret_cast<S *>(smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u));

  // The rescan of a cut sequence is a programmatic dependent of the carry,
  // whose entering states every segment reads: its CTAs are placed while
  // the carry runs and wait here for it.
  if (MODE == kModeFull && p.nseg > 1) pdl_wait();
  const int64_t L = p.L, C = p.C, Gr = p.G;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ch = lane / G, q = lane % G;
  const int cw0 = warp * CPW;  // the warp's first channel within the CTA's 32
  const int64_t c0 = (int64_t)blockIdx.x * kCT;
  const int64_t c = c0 + cw0 + ch;
  const bool cvalid = c < C;
  const int b = blockIdx.y;
  const int seg = blockIdx.z;
  const int g = (int)(c0 / (C / Gr));
  constexpr bool rms_bc = RBC;  // the host picks the instance from SSM_RMSNORM_BC
  // A state written at token t (p.state_write): tokens before t do not see
  // it and tokens after t see only it, so the call is three independent
  // parts -- 0: tokens [0, t) from h0; 1: token t's readout; 2: tokens
  // (t, L) from the written state, which leave h_last -- taken by the grid's
  // third dimension from p.part_base on (one launch, or two when h_last
  // overlaps what parts 0 and 1 read).
  const bool wsplit = kFull && p.state_write != nullptr;
  const int part = p.part_base + seg;
  int64_t tb, te;
  if (wsplit) {
    tb = part == 0 ? 0 : p.t_write + 1;
    te = part == 0 ? p.t_write : L;
  } else {
    tb = (int64_t)seg * p.seg_len;
    te = tb + p.seg_len < L ? tb + p.seg_len : L;
  }
  if (wsplit && part == 1) {
    // y_t = C_t . (written state), with the chain's arithmetic: the same
    // per-lane partials and reduction (its pairing does not depend on the
    // token's place in a group), C_t's factor formed as the prologue forms
    // it, the skip term and the gate -- so y_t is the one a scan whose
    // state at t is the written one gives.  Every lane takes part in the
    // shuffles; lanes past the last channel store nothing.
    const int64_t t = p.t_write;
    const T *Cg = static_cast<const T *>(p.Cm) + ((b * L + t) * Gr + g) * N;
    f2 hw[NP], cv[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) hw[j] = mk2(0.f, 0.f);
    if (cvalid) load_pairs<NP>(p.state_write + (b * C + c) * N + SPL * q, hw);
    load_pairs_io<NP>(Cg + SPL * q, cv);
    f2 acc = mul2(cv[0], hw[0]);
#pragma unroll
    for (int j = 1; j < NP; ++j) acc = fma2(cv[j], hw[j], acc);
    float pg[G];
#pragma unroll
    for (int u = 0; u < G; ++u) pg[u] = acc.x + acc.y;
    const float yq = transpose_reduce<G>(pg, q);
    float rc = 1.f;
    if constexpr (rms_bc) {
      constexpr int PN = N / 4;
      float vc[PN];
      widen<PN>(Cg + (lane & 3) * PN, vc);
      float sc = 0.f;
#pragma unroll
      for (int i = 0; i < PN; ++i) sc = fmaf(vc[i], vc[i], sc);
      sc += __shfl_xor_sync(0xffffffffu, sc, 1);
      sc += __shfl_xor_sync(0xffffffffu, sc, 2);
      rc = rsqrtf(sc / N + p.eps);
    }
    if (cvalid && q == 0) {
      const int64_t i = (b * L + t) * C + c;
      const float dx = (p.D ? p.D[c] : 0.f) * ld(static_cast<const T *>(p.x) + i);
      float gate = 1.f;
      if (HAS_Z) {
        const float zv = ld(static_cast<const T *>(p.z) + i);
        gate = kBF16 ? silu_tanh(zv) : silu(zv);
      }
      const float v = rms_bc ? fmaf(yq, rc, dx) : yq + dx;
      st(static_cast<T *>(p.y) + i, v * gate);
    }
    return;
  }
  const int nst = (int)((te - tb + kTL - 1) / kTL);
  const bool softplus_on = p.flags & 1u;
  constexpr uint32_t kStageBytes = ((HAS_Z ? 3 : 2) * kTL * kCT + 2 * kTL * N) * sizeof(T);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.conv[i], NW * 32);  // every lane arrives (release of its own writes)
      mbar_init(&s.empty[i], NW * 32);
    }
    mbar_init(&s.ylast, NW * 32);
    fence_mbar_init();
  }
  if (threadIdx.x < kCT) {
    const bool v = c0 + threadIdx.x < C;
    s.bias[threadIdx.x] = (p.dt_bias && v) ? p.dt_bias[c0 + threadIdx.x] : 0.f;
    s.skip[threadIdx.x] = (p.D && v) ? p.D[c0 + threadIdx.x] : 0.f;
  }
  __syncthreads();

  const bool issuer = threadIdx.x == 0;
  int issued = 0;
  // No L2 policy on these loads: an evict-first hint on the streamed x, dt, z
  // boxes (64 B of each 128-B line per CTA) let L2 drop a line after one
  // channel block had read its half and before its neighbour read the other,
  // which then came from DRAM again (a quarter more reads at the Falcon
  // width), and evict-last on B and C gained nothing measurable.
  auto issue = [&](int stage) {
    const int buf = stage % NS;
    const int t0 = (int)(tb + (int64_t)stage * kTL);
    mbar_expect_tx(&s.full[buf], kStageBytes);
    tma_load_3d(&s.x[buf][0][0], &mx, &s.full[buf], (int)c0, t0, b);
    tma_load_3d(&s.dt[buf][0][0], &mdt, &s.full[buf], (int)c0, t0, b);
    if (HAS_Z) tma_load_3d(&s.z[buf][0][0], &mz, &s.full[buf], (int)c0, t0, b);
    tma_load_3d(&s.B[buf][0][0], &mB, &s.full[buf], g * N, t0, b);
    tma_load_3d(&s.C[buf][0][0], &mC, &s.full[buf], g * N, t0, b);
  };
  if (issuer)
    for (; issued < NS && issued < nst; ++issued) issue(issued);

  // The start state: h0 (or zeros), the carried state of this segment, or
  // zeros for a segment scanned from its own start.
  const float *h_in = nullptr;
  if (MODE == kModeStateOnly) h_in = seg == 0 ? p.h0 : nullptr;
  else if (wsplit) h_in = part == 0 ? p.h0 : p.state_write;
  else h_in = p.nseg > 1 ? p.seg_ent + (int64_t)seg * p.batch * C * N : p.h0;
  f2 h[NP], A2[NP];
#pragma unroll
  for (int j = 0; j < NP; ++j) h[j] = A2[j] = mk2(0.f, 0.f);
  if (cvalid) {
    if (h_in) load_pairs<NP>(h_in + (b * C + c) * N + SPL * q, h);
    load_pairs<NP>(p.A + c * N + SPL * q, A2);
#pragma unroll
    for (int j = 0; j < NP; ++j) A2[j] = mk2(A2[j].x * kLog2e, A2[j].y * kLog2e);
  }
  // The FMA-pipe exponential assumes decays (d >= 0, A < 0); a warp where any
  // of its states could grow keeps every decay on the SFU.
  // (the last pair of a lane's states, when PX == 2)
  const f2 Al = A2[NP - 1];
  const f2 liml = mk2(Al.x < 0.f ? -127.f / Al.x : 3.0e38f, Al.y < 0.f ? -127.f / Al.y : 3.0e38f);
  const bool poly_ok =
      PX == 2 && __all_sync(0xffffffffu, softplus_on && ((Al.x < 0.f && Al.y < 0.f) || !cvalid));
  float dsum = 0.f;
  bool failed = false;
  // The prologue's lane always takes the same 8 channels (k0 below): their
  // step bias and skip weight stay in registers.
  float biasr[8], skipr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    biasr[i] = s.bias[(lane & 3) * 8 + i];
    skipr[i] = s.skip[(lane & 3) * 8 + i];
  }
  // Rows [warp * kTL / NW, + kTL / NW) of stage st's y staging (token t0y
  // onwards, tny of them in the segment) to global memory, 16 bytes a lane.
  auto store_y = [&](int st, int64_t t0y, int tny) {
    constexpr int kRows = kTL / NW;
    constexpr int kChunks = kCT * (int)sizeof(T) / 16;  // per row
    char *yg = static_cast<char *>(p.y);
    for (int e = lane; e < kRows * kChunks; e += 32) {
      const int t = warp * kRows + e / kChunks, k = e % kChunks;
      const int64_t cg = c0 + (int64_t)k * 16 / (int64_t)sizeof(T);  // chunk's first channel
      if (t >= tny || cg >= C) continue;  // C is a multiple of 16 bytes' worth
      *reinterpret_cast<uint4 *>(yg + ((b * L + t0y + t) * C + cg) * (int64_t)sizeof(T)) =
          *reinterpret_cast<const uint4 *>(reinterpret_cast<const char *>(&s.y[st & 1][t][0]) + 16 * k);
    }
  };

  for (int sg = 0; sg < nst; ++sg) {
    const int buf = sg % NS;
    const uint32_t ph = (uint32_t)(sg / NS) & 1u;
    const int64_t t0 = tb + (int64_t)sg * kTL;
    const int tn = (int)(te - t0 < kTL ? te - t0 : kTL);  // tokens of this segment in the stage
    if (!__all_sync(0xffffffffu, mbar_wait(&s.full[buf], ph, kWaitLimit))) {
      failed = true;
      break;
    }
    // ---- 2. per (token, channel) of this warp's tokens, all 32 channels:
    // d = softplus(dt * rstd + bias), d * x, D * x and the gate factor.  Four
    // lanes share a token, each taking 8 channels (conflict-free 16-byte rows).
    // With RMS norms on B and C the four also form the token's two factors
    // 1 / rms over the state (a quarter of B_t and C_t each, summed across
    // the four): B_t's multiplies d * x, so that the recurrence's write term
    // d x (B_t / rms(B_t)) needs B_t only as it landed; C_t's is kept for the
    // readout, which scales the reduced C_t . h once.  The recurrence reads
    // B and C as bfloat16 straight from the stage either way.
    for (int e = lane; e < TPW * 4; e += 32) {
      const int t = warp * TPW + (e >> 2), k0 = (e & 3) * 8;
      const bool tvalid = t < tn;
      const float rs = (tvalid && p.rstd) ? p.rstd[b * L + t0 + t] : 1.f;
      float rb = 1.f;
      if constexpr (rms_bc) {
        constexpr int PN = N / 4;  // values of B_t (and of C_t) per lane of the four
        // (a token's four lanes are all in the loop or all out of it)
        const unsigned quad = 0xfu << (lane & 28);
        float vb[PN], vc[PN];
        widen<PN>(&s.B[buf][t][(e & 3) * PN], vb);
        widen<PN>(&s.C[buf][t][(e & 3) * PN], vc);
        float sb = 0.f, sc = 0.f;
#pragma unroll
        for (int i = 0; i < PN; ++i) {
          sb = fmaf(vb[i], vb[i], sb);
          sc = fmaf(vc[i], vc[i], sc);
        }
        sb += __shfl_xor_sync(quad, sb, 1);
        sc += __shfl_xor_sync(quad, sc, 1);
        sb += __shfl_xor_sync(quad, sb, 2);
        sc += __shfl_xor_sync(quad, sc, 2);
        rb = rsqrtf(sb / N + p.eps);
        if ((e & 3) == 0) s.rc[sg & 1][t] = rsqrtf(sc / N + p.eps);
      }
      float xv[8], dv[8], zv[8];
      widen<8>(&s.x[buf][t][k0], xv);
      widen<8>(&s.dt[buf][t][k0], dv);
      if (HAS_Z) widen<8>(&s.z[buf][t][k0], zv);
      // channel pairs in packed f32x2 where the scalar form is one
      // operation per channel (each lane exactly that operation)
      float2 o[8], og[8];
      const f2 rs2 = mk2(rs, rs), rb2 = mk2(rb, rb);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = 2 * k;
        const f2 x2 = mk2(xv[i], xv[i + 1]);
        f2 d2 = fma2(mk2(dv[i], dv[i + 1]), rs2, mk2(biasr[i], biasr[i + 1]));
        if (softplus_on) d2 = mk2(softplus_sfu(d2.x), softplus_sfu(d2.y));
        const f2 dx2 = mul2(mul2(d2, x2), rb2);
        const f2 sx2 = mul2(mk2(skipr[i], skipr[i + 1]), x2);
        f2 g2 = mk2(1.f, 1.f);
        if (HAS_Z) {
          if (kBF16) {  // silu(z) = z (1 + tanh(z / 2)) / 2, as silu_tanh
            const f2 z2 = mk2(zv[i], zv[i + 1]);
            const f2 hz = mul2(mk2(0.5f, 0.5f), z2);
            float ta, tb;
            asm("tanh.approx.f32 %0, %1;" : "=f"(ta) : "f"(hz.x));
            asm("tanh.approx.f32 %0, %1;" : "=f"(tb) : "f"(hz.y));
            g2 = mul2(z2, fma2(mk2(0.5f, 0.5f), mk2(ta, tb), mk2(0.5f, 0.5f)));
          } else {
            g2 = mk2(silu(zv[i]), silu(zv[i + 1]));
          }
        }
        o[i] = tvalid ? make_float2(d2.x, dx2.x) : make_float2(0.f, 0.f);
        o[i + 1] = tvalid ? make_float2(d2.y, dx2.y) : make_float2(0.f, 0.f);
        og[i] = make_float2(sx2.x, g2.x);
        og[i + 1] = make_float2(sx2.y, g2.y);
      }
      float4 *dst = reinterpret_cast<float4 *>(&s.ddx[sg & 1][t][k0]);
      float4 *gst = reinterpret_cast<float4 *>(&s.eg[sg & 1][t][k0]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dst[i] = make_float4(o[2 * i].x, o[2 * i].y, o[2 * i + 1].x, o[2 * i + 1].y);
        gst[i] = make_float4(og[2 * i].x, og[2 * i].y, og[2 * i + 1].x, og[2 * i + 1].y);
      }
    }
    mbar_arrive(&s.conv[buf]);
    if (!__all_sync(0xffffffffu, mbar_wait(&s.conv[buf], ph, kWaitLimit))) {
      failed = true;
      break;
    }

    // ---- 3. the recurrence.  Tokens go in steps of SL; the decays and
    // write terms of step k+1 (independent of the state) are formed while
    // step k runs its chain, and the readout of step k-1 is reduced and
    // stored meanwhile, so that a warp always has independent work at hand.
    // (8 tokens per step: measured 8 % faster than 4 at the Falcon width,
    // equal on the 130m workload; 16 is slower.)
    constexpr int SL = G > 8 ? G : 8;  // tokens per step
    struct Pre {
      f2 a[SL][NP], w[SL][NP];  // decays and write terms d * x * B
    };
    auto pre = [&](int tg, Pre &P) {
#pragma unroll
      for (int u = 0; u < SL; ++u) {
        const int t = tg + u;
        const float2 dd = s.ddx[sg & 1][t][cw0 + ch];
        f2 bv[NP];
        load_pairs_io<NP>(&s.B[buf][t][SPL * q], bv);
        const f2 d2 = mk2(dd.x, dd.x), dx2 = mk2(dd.y, dd.y);
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          if (j == NP - 1 && poly_ok) {
            P.a[u][j] = exp2_fma2(dd.x, Al, liml);
          } else {
            const f2 dA = mul2(d2, A2[j]);
            P.a[u][j] = mk2(ex2(dA.x), ex2(dA.y));
          }
          P.w[u][j] = mul2(dx2, bv[j]);
        }
        if (!kFull) dsum += dd.x;
      }
    };
    // y for the tokens of one step from its partials (lane q of each group
    // of G lanes finishes token tg + G k + q)
    auto finish = [&](int tg, float (&part)[SL]) {
#pragma unroll
      for (int k = 0; k < SL / G; ++k) {
        float pg[G];
#pragma unroll
        for (int u = 0; u < G; ++u) pg[u] = part[G * k + u];
        const float yq = transpose_reduce<G>(pg, q);
        const int tt = tg + G * k + q;
        const float2 eg = s.eg[sg & 1][tt][cw0 + ch];
        const float ch_ = rms_bc ? fmaf(yq, s.rc[sg & 1][tt], eg.x) : yq + eg.x;
        st(&s.y[sg & 1][tt][cw0 + ch], ch_ * eg.y);
      }
    };
    Pre cur, nxt;
    pre(0, cur);
    float partp[SL];
#pragma unroll
    for (int tg = 0; tg < kTL; tg += SL) {
      if (tg + SL < kTL) pre(tg + SL, nxt);
      float part[SL];
      // the chain of one step
#pragma unroll
      for (int u = 0; u < SL; ++u) {
        const int t = tg + u;
#pragma unroll
        for (int j = 0; j < NP; ++j) h[j] = fma2(cur.a[u][j], h[j], cur.w[u][j]);
        if (kFull) {
          f2 cv[NP];
          load_pairs_io<NP>(&s.C[buf][t][SPL * q], cv);
          f2 acc = mul2(cv[0], h[0]);
#pragma unroll
          for (int j = 1; j < NP; ++j) acc = fma2(cv[j], h[j], acc);
          part[u] = acc.x + acc.y;
        }
        if (STATES && cvalid && t < tn)
          store_pairs<NP>(p.states + ((b * L + t0 + t) * C + c) * N + SPL * q, h);
      }
      if (kFull && tg >= SL) finish(tg - SL, partp);
#pragma unroll
      for (int u = 0; u < SL; ++u) partp[u] = part[u];
      cur = nxt;
    }
    if (kFull) finish(kTL - SL, partp);
    mbar_arrive(&s.empty[buf]);
    // ---- 4. y of the previous stage: every warp has finished it (they all
    // arrived on this stage's `conv`), so this warp stores its share of the
    // rows, after its own recurrence (measured: 2 % faster than storing them
    // before it, 5 % faster than each warp storing its own 16-byte rows)
    if (kFull && sg >= 1) store_y(sg - 1, t0 - kTL, kTL);

    // ---- refill the buffer of the previous stage once every warp left it
    if (issuer && sg >= 1 && issued < nst) {
      const int prev = sg - 1;
      if (!mbar_wait(&s.empty[prev % NS], (uint32_t)(prev / NS) & 1u, kWaitLimit)) {
        failed = true;
      } else {
        issue(issued);
        ++issued;
      }
    }
    if (__any_sync(0xffffffffu, failed)) break;
  }

  // y of the last stage, once every warp has written it
  if (kFull && !failed && nst > 0) {
    mbar_arrive(&s.ylast);
    if (__all_sync(0xffffffffu, mbar_wait(&s.ylast, 0, kWaitLimit))) {
      const int64_t tl = tb + (int64_t)(nst - 1) * kTL;
      store_y(nst - 1, tl, (int)(te - tl));
    } else {
      failed = true;
    }
  }
  if (failed) {
    if (lane == 0 && p.status) atomicExch(p.status, 1);
    // let every copy this CTA started land before its shared memory goes
    if (issuer)
      for (int st_ = 0; st_ < issued; ++st_)
        mbar_wait(&s.full[st_ % NS], (uint32_t)(st_ / NS) & 1u, kWaitLimit);
    return;
  }
  if (!cvalid) return;
  if (MODE == kModeStateOnly) {
    const int64_t i = ((int64_t)seg * p.batch + b) * C + c;
    store_pairs<NP>(p.seg_end + i * N + SPL * q, h);
    if (q == 0) p.seg_dsum[i] = dsum;
  } else if (p.h_last && (wsplit ? part == 2 : seg == p.nseg - 1)) {
    store_pairs<NP>(p.h_last + (b * C + c) * N + SPL * q, h);
  }
}

// The carry between segments: for each (batch, channel, state) the states
// entering segments 1..S-1 from the end states of segments 0..S-2 (segment 0
// from h0, the others from zeros) and the decay products
// P_k = exp(A * sum of segment k's steps).  Pairs (P, E) compose as
// (P_a, E_a) then (P_b, E_b) = (P_a P_b, P_b E_a + E_b); an inclusive
// shuffle scan over a group of SP lanes (lane k = segment k) gives each
// segment's entering state.  Also copies h0 (or zeros) as segment 0's
// entering state, so that the rescan never reads h0 (which h_last may alias).
template <int SP>
__global__ void m1_seg_carry_kernel(const M1Params p) {
  pdl_launch_dependents();  // the rescan's CTAs may be placed (they wait for this launch)
  const int64_t items = p.batch * p.C * p.N;
  const int64_t idx = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / SP;
  const int k = threadIdx.x % SP;
  const bool live = idx < items;
  const int64_t it = live ? idx : 0;
  const int64_t n = it % p.N, bc = it / p.N, c = bc % p.C;
  const int nprev = p.nseg - 1;  // segments with an end state
  float P = 1.f, E = 0.f;
  if (live && k < nprev) {
    E = p.seg_end[(int64_t)k * items + it];
    if (k > 0) P = ex2(p.A[c * p.N + n] * kLog2e * p.seg_dsum[(int64_t)k * p.batch * p.C + bc]);
  }
#pragma unroll
  for (int o = 1; o < SP; o <<= 1) {
    const float Pp = __shfl_up_sync(0xffffffffu, P, o, SP);
    const float Ep = __shfl_up_sync(0xffffffffu, E, o, SP);
    if (k >= o) {
      E = fmaf(P, Ep, E);
      P *= Pp;
    }
  }
  if (!live) return;
  if (k < nprev) p.seg_ent[(int64_t)(k + 1) * items + it] = E;
  if (k == 0) p.seg_ent[it] = p.h0 ? p.h0[it] : 0.f;
}

template <typename T>
CUtensorMapDataType tmap_type() {
  return sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
}

struct Maps {
  CUtensorMap x, dt, z, B, C;
};

template <int N, typename T>
bool make_maps(const M1Params &p, Maps &m) {
  const uint64_t es = sizeof(T);
  uint64_t dims[3] = {(uint64_t)p.C, (uint64_t)p.L, (uint64_t)p.batch};
  uint64_t strides[2] = {(uint64_t)p.C * es, (uint64_t)(p.L * p.C) * es};
  uint32_t box[3] = {(uint32_t)kCT, (uint32_t)kTL, 1};
  if (!encode_tiled(&m.x, tmap_type<T>(), 3, p.x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tiled(&m.dt, tmap_type<T>(), 3, p.dt, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  if (p.z) {
    if (!encode_tiled(&m.z, tmap_type<T>(), 3, p.z, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  } else {
    m.z = m.x;
  }
  const uint64_t GN = (uint64_t)(p.G * p.N);
  uint64_t bdims[3] = {GN, (uint64_t)p.L, (uint64_t)p.batch};
  uint64_t bstrides[2] = {GN * es, (uint64_t)p.L * GN * es};
  uint32_t bbox[3] = {(uint32_t)N, (uint32_t)kTL, 1};
  return encode_tiled(&m.B, tmap_type<T>(), 3, p.B, bdims, bstrides, bbox,
                      CU_TENSOR_MAP_SWIZZLE_NONE) &&
         encode_tiled(&m.C, tmap_type<T>(), 3, p.Cm, bdims, bstrides, bbox,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int N, int SPL, typename T, bool HZ, int MODE, bool ST>
cudaError_t launch_spl(const Maps &m, const M1Params &p, int nseg, cudaStream_t s,
                       bool dependent) {
  constexpr int NS = 3;
  auto k = (p.flags & 2u) ? m1_scan_tma_kernel<N, SPL, T, NS, HZ, MODE, ST, kPolyStates, true>
                          : m1_scan_tma_kernel<N, SPL, T, NS, HZ, MODE, ST, kPolyStates, false>;
  const size_t smem = sizeof(ScanSmem<N, T, NS>) + 128;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.C + kCT - 1) / kCT), (unsigned)p.batch, (unsigned)nseg);
  if (dependent)
    return launch_dependent(k, grid, dim3(kCT * (N / SPL)), smem, s, m.x, m.dt, m.z, m.B, m.C, p);
  k<<<grid, kCT * (N / SPL), smem, s>>>(m.x, m.dt, m.z, m.B, m.C, p);
  return cudaGetLastError();
}

// Four states per lane.  (Two per lane doubles the warps but, measured on
// the 130m workload, costs 66 % more instructions per state and runs 24 %
// slower: the transposing reduction spans eight lanes and every B/C load
// serves half as many states.)
template <int N, typename T, bool HZ, int MODE, bool ST>
cudaError_t launch_one(const Maps &m, const M1Params &p, int nseg, cudaStream_t s,
                       bool dependent = false) {
  return launch_spl<N, 4, T, HZ, MODE, ST>(m, p, nseg, s, dependent);
}

template <int N, typename T, bool HZ>
cudaError_t launch_n(const M1Params &p, cudaStream_t s) {
  Maps m;
  if (!make_maps<N, T>(p, m)) return cudaErrorInvalidValue;
  if (p.states) return launch_one<N, T, HZ, kModeFull, true>(m, p, 1, s);
  if (p.state_write) {
    // three independent parts in one launch (see the kernel), unless h_last
    // overlaps h0 or the written state: part 2 writes h_last, which parts 0
    // and 1 read, so it then runs as a launch of its own after theirs
    const size_t n = (size_t)(p.batch * p.C * p.N) * sizeof(float);
    auto overlap = [n](const void *a, const void *b) {
      const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
      return a && b && x < y + n && y < x + n;
    };
    if (!overlap(p.h_last, p.h0) && !overlap(p.h_last, p.state_write))
      return launch_one<N, T, HZ, kModeFull, false>(m, p, 3, s);
    M1Params q = p;
    q.part_base = 0;
    cudaError_t e = launch_one<N, T, HZ, kModeFull, false>(m, q, 2, s);
    if (e != cudaSuccess) return e;
    q.part_base = 2;
    return launch_one<N, T, HZ, kModeFull, false>(m, q, 1, s);
  }
  if (p.nseg <= 1) return launch_one<N, T, HZ, kModeFull, false>(m, p, 1, s);
  cudaError_t e = launch_one<N, T, HZ, kModeStateOnly, false>(m, p, p.nseg - 1, s);
  if (e != cudaSuccess) return e;
  const int64_t items = p.batch * p.C * p.N;
  const int sp = p.nseg - 1 <= 2 ? 2 : p.nseg - 1 <= 4 ? 4 : p.nseg - 1 <= 8 ? 8 : p.nseg - 1 <= 16 ? 16 : 32;
  const unsigned blocks = (unsigned)((items * sp + 255) / 256);
  switch (sp) {
    case 2: m1_seg_carry_kernel<2><<<blocks, 256, 0, s>>>(p); break;
    case 4: m1_seg_carry_kernel<4><<<blocks, 256, 0, s>>>(p); break;
    case 8: m1_seg_carry_kernel<8><<<blocks, 256, 0, s>>>(p); break;
    case 16: m1_seg_carry_kernel<16><<<blocks, 256, 0, s>>>(p); break;
    default: m1_seg_carry_kernel<32><<<blocks, 256, 0, s>>>(p); break;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_one<N, T, HZ, kModeFull, false>(m, p, p.nseg, s, true);
}

template <typename T>
cudaError_t launch_t(const M1Params &p, cudaStream_t s) {
  const bool hz = p.z != nullptr;
  switch (p.N) {
    case 4:
      if constexpr (sizeof(T) == 4) return hz ? launch_n<4, T, true>(p, s) : launch_n<4, T, false>(p, s);
      break;
    case 8: return hz ? launch_n<8, T, true>(p, s) : launch_n<8, T, false>(p, s);
    case 16: return hz ? launch_n<16, T, true>(p, s) : launch_n<16, T, false>(p, s);
    case 32: return hz ? launch_n<32, T, true>(p, s) : launch_n<32, T, false>(p, s);
  }
  return cudaErrorNotSupported;
}

}  // namespace

// The pipelined kernel needs 16-byte rows for TMA (x/dt/z rows of the tensor
// and B/C rows of one group), 32-channel tiles inside one B/C group, and
// N in {8, 16, 32} (N = 4 for float32 I/O).
bool m1_scan_tma_supported(const M1Params &p) {
  const int64_t es = p.io == 1 ? 2 : 4;
  const bool n_ok = p.N == 8 || p.N == 16 || p.N == 32 || (p.N == 4 && es == 4);
  if (!n_ok) return false;
  if ((p.N * es) % 16 || (p.C * es) % 16 || (p.G * p.N * es) % 16) return false;
  if (p.G > 1 && (p.C / p.G) % kCT) return false;
  if (p.L >= (1ll << 31) || p.C >= (1ll << 31) || p.batch > 65535) return false;
  return true;
}

// How many sequence segments a call is cut into.  Cost model (measured on
// B200 for this kernel, 16 states): a warp's time per token with k warps on
// its SM sub-partition is flat, ~79 ns, up to about two warps (the chain is
// latency-bound there), then the sub-partition's issue and SFU throughput is
// shared, ~33.5 k ns.  A pass of W warps over Ls tokens takes
// Ls * t(ceil(W / sub-partitions)).  Cutting into S segments costs a
// state-only pass over the first S - 1 segments (about 0.85 of a full pass
// per token, no readout), a full pass over S segments of 1/S of the sequence
// each, and ~14 us of fills, carry and launches.  A cut is taken when it is
// predicted 10 % faster.  Calls with per-token states or a state write are
// not cut.
M1Split m1_scan_split(int64_t batch, int64_t C, int64_t L, int64_t N, int sms) {
  M1Split r;
  r.nseg = 1;
  r.seg_len = L;
  if (batch <= 0 || L <= 0 || sms <= 0) return r;
  const double kStateOnly = 0.85, kCutNs = 14000.0;
  const double slots = 4.0 * sms;  // sub-partitions
  const double w0 = (double)batch * ((C + kCT - 1) / kCT) * (kCT * (N / 4) / 32);  // warps
  auto pass_ns = [&](double warps, double tokens) {
    const double k = std::ceil(warps / slots);
    return tokens * std::max(79.0, 33.5 * k);
  };
  double best = pass_ns(w0, (double)L);
  for (int S = 2; S <= 32; S *= 2) {
    const int64_t len = ((L + S - 1) / S + kTL - 1) / kTL * kTL;
    if (len < 4 * kTL) break;
    const int segs = (int)((L + len - 1) / len);
    if (segs < 2) break;
    const double t = kStateOnly * pass_ns(w0 * (segs - 1), (double)len) +
                     pass_ns(w0 * segs, (double)len) + kCutNs;
    if (t < 0.9 * best) {
      best = t;
      r.nseg = segs;
      r.seg_len = len;
    }
  }
  return r;
}

size_t m1_scan_split_bytes(const M1Split &r, int64_t batch, int64_t C, int64_t N) {
  if (r.nseg <= 1) return 0;
  const size_t bcn = (size_t)(batch * C * N) * sizeof(float);
  const size_t bc = (size_t)(batch * C) * sizeof(float);
  const auto a16 = [](size_t v) { return (v + 255) & ~(size_t)255; };
  return a16(bcn * (r.nseg - 1)) + a16(bc * (r.nseg - 1)) + a16(bcn * r.nseg);
}

void m1_scan_split_carve(const M1Split &r, int64_t batch, int64_t C, int64_t N, void *ws,
                         M1Params &p) {
  p.nseg = r.nseg;
  p.seg_len = r.seg_len;
  if (r.nseg <= 1) return;
  const size_t bcn = (size_t)(batch * C * N) * sizeof(float);
  const size_t bc = (size_t)(batch * C) * sizeof(float);
  const auto a16 = [](size_t v) { return (v + 255) & ~(size_t)255; };
  char *w = static_cast<char *>(ws);
  p.seg_end = reinterpret_cast<float *>(w);
  w += a16(bcn * (r.nseg - 1));
  p.seg_dsum = reinterpret_cast<float *>(w);
  w += a16(bc * (r.nseg - 1));
  p.seg_ent = reinterpret_cast<float *>(w);
}

cudaError_t launch_m1_scan_tma(const M1Params &p, cudaStream_t s) {
  return p.io == 1 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace ssm
