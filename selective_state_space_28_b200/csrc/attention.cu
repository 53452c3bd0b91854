// attention.cu -- the hidden attention of the Mamba-2 (SSD) map ("Mamba-2",
// nnterp encyclopedia, "The hidden attention"): per head the causal
// [seq, seq] matrix
//
//   alpha[t, s] = (C_t . B_s) * exp(decays_{s+1} + ... + decays_t) * betas_s
//
// for s <= t (zero above the diagonal), with betas = softplus(dt + dt_bias)
// and decays = betas * A_h, so that y_t = sum_s alpha[t, s] x_s + D x_t from
// a zero state.
//
// Writing b * H * L^2 float32 values dominates; C . B^T does not depend on the
// head, so one pass computes each 128 x 128 tile of it on or below the
// diagonal once per (batch, group) into the workspace (where it stays in L2;
// on the tensor cores for bf16 inputs with state 128, else on the CUDA cores),
// and the mask pass -- one CTA per (query tile, key tile, four heads of the
// group) -- reads its share of the tile once and applies each head's decay
// mask to it.  The decay between s and t is taken as the
// difference of a running sum kept in float64 (a pre-pass), so that long
// sequences lose no precision to the cancellation.  Below the diagonal 32 x 32
// blocks the factor exp(cum_t - cum_s) is split at the last key r of s's
// 32-token block into exp(cum_t - cum_r) * exp(cum_r - cum_s), both <= 1 for
// a decaying state; on the diagonal blocks it is taken element by element.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma.h"

#include <type_traits>

namespace ssm {
namespace {

using namespace sm100;

constexpr int kTile = 128;   // query and key tokens per tile
constexpr int kHeadsPerCta = 4;

// Pre-pass: per (batch, head) the step betas_t and the running sum of the
// log2-decays, cum_t = sum_{r <= t} betas_r A_h log2(e), in float64.  One
// block per (batch, head), kPrep tokens per round: each thread loads one
// token, and a block-wide scan (warp shuffles, then the warps' totals)
// gives the running sums.
constexpr int kPrep = 1024;
template <typename T>
__global__ void __launch_bounds__(kPrep) attn_prep_kernel(AttnParams p) {
  __shared__ double wsum[kPrep / 32];
  const int64_t unit = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t b = unit / p.H, h = unit % p.H;
  const T *dt = static_cast<const T *>(p.dt);
  const double A2 = (double)p.A[h] * 1.4426950408889634;
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
  double carry = 0.0;
  for (int64_t t0 = 0; t0 < p.L; t0 += kPrep) {
    const int64_t t = t0 + tid;
    float d = 0.f;
    if (t < p.L) {
      d = ld(dt + (b * p.L + t) * p.H + h) + bias;
      if (p.flags & 1u) d = softplus(d);
    }
    double v = (double)d * A2;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    double before = carry, total = carry;
    for (int w = 0; w < kPrep / 32; ++w) {
      const double x = wsum[w];
      if (w < warp) before += x;
      total += x;
    }
    if (t < p.L) {
      p.beta[unit * p.L + t] = d;
      p.cum[unit * p.L + t] = before + v;
    }
    carry = total;
    __syncthreads();  // wsum is rewritten next round
  }
}

// Tile index of query tile qt, key tile kt <= qt in the packed lower
// triangle of tiles.
__device__ __forceinline__ int64_t lower_index(int64_t qt, int64_t kt) {
  return qt * (qt + 1) / 2 + kt;
}

// C . B^T for every tile on or below the diagonal, once per (batch, group):
// sixteen CTAs per tile, one per 32 x 32 block, each staging its 32 query and
// 32 key rows of C and B over the whole state axis in one load (for state up
// to 128; longer states take more passes).  256 threads: thread (ty, tx)
// owns row ty and columns 4 tx .. 4 tx + 3 of the block.  The tile goes to
// the workspace (float32, rows of 128), where it stays in L2 for the mask
// pass.
constexpr int kBlk = 32;
constexpr int kKc = 128;     // state columns per pass
constexpr int kBPitch = 36;  // floats per row of the k-major staging (16-byte rows)
template <typename T>
__global__ void __launch_bounds__(256) attn_cb_kernel(AttnParams p) {
  __shared__ __align__(16) float Cs[kKc][kBPitch];  // [k][query]
  __shared__ __align__(16) float Bs[kKc][kBPitch];  // [k][key]
  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  const int64_t L = p.L;
  // blockIdx.x enumerates (packed lower triangle of tiles) x (16 blocks)
  const int64_t li = blockIdx.x >> 4;
  const int blk = blockIdx.x & 15, br = blk >> 2, bc = blk & 3;
  int64_t qt = (int64_t)((sqrt(8.0 * (double)li + 1.0) - 1.0) / 2.0);
  while (qt * (qt + 1) / 2 > li) --qt;
  while ((qt + 1) * (qt + 2) / 2 <= li) ++qt;
  const int64_t kt = li - qt * (qt + 1) / 2;
  const int64_t t0 = qt * kTile + br * kBlk, s0 = kt * kTile + bc * kBlk;
  const int64_t g = blockIdx.y, b = blockIdx.z;
  const T *Cg = static_cast<const T *>(p.Cm);
  const T *Bg = static_cast<const T *>(p.B);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t k0 = 0; k0 < p.N; k0 += kKc) {
    for (int e = tid; e < kBlk * kKc; e += 256) {
      const int r = e / kKc, k = e % kKc;
      const int64_t tq = t0 + r, tk = s0 + r;
      const bool kin = k0 + k < p.N;
      Cs[k][r] = (tq < L && kin) ? ld(Cg + ((b * L + tq) * p.G + g) * p.N + k0 + k) : 0.f;
      Bs[k][r] = (tk < L && kin) ? ld(Bg + ((b * L + tk) * p.G + g) * p.N + k0 + k) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kKc; ++k) {
      const float a = Cs[k][ty];
      const float4 c4 = *reinterpret_cast<const float4 *>(&Bs[k][4 * tx]);
      acc[0] = fmaf(a, c4.x, acc[0]);
      acc[1] = fmaf(a, c4.y, acc[1]);
      acc[2] = fmaf(a, c4.z, acc[2]);
      acc[3] = fmaf(a, c4.w, acc[3]);
    }
    __syncthreads();
  }
  float *tile = p.cb + ((b * p.G + g) * p.ntri + li) * (int64_t)(kTile * kTile);
  *reinterpret_cast<float4 *>(tile + (br * kBlk + ty) * kTile + bc * kBlk + 4 * tx) =
      make_float4(acc[0], acc[1], acc[2], acc[3]);
}

// The pre-pass's running sums for one (batch, head) with 128 threads (the
// pre-pass blocks of the fused launch below): per 1024-token round each
// thread loads 8 consecutive tokens and sums them in order; a block-wide scan
// of the threads' totals (warp shuffles, then the four warps' totals) gives
// every token's running sum.
constexpr int kPrepSmall = 128, kPrepRun = 8;
template <typename T>
__device__ __forceinline__ void prep_unit_small(const AttnParams &p, int64_t unit) {
  __shared__ double wsum[kPrepSmall / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t b = unit / p.H, h = unit % p.H;
  const T *dt = static_cast<const T *>(p.dt);
  const double A2 = (double)p.A[h] * 1.4426950408889634;
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
  double carry = 0.0;
  for (int64_t t0 = 0; t0 < p.L; t0 += kPrepSmall * kPrepRun) {
    const int64_t tb = t0 + (int64_t)tid * kPrepRun;
    float d[kPrepRun];
#pragma unroll
    for (int j = 0; j < kPrepRun; ++j) {
      d[j] = 0.f;
      if (tb + j < p.L) {
        d[j] = ld(dt + (b * p.L + tb + j) * p.H + h) + bias;
        if (p.flags & 1u) d[j] = softplus(d[j]);
      }
    }
    double run[kPrepRun], v = 0.0;
#pragma unroll
    for (int j = 0; j < kPrepRun; ++j) {
      v += (double)d[j] * A2;
      run[j] = v;  // within the thread's 8 tokens
    }
    double incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double u = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += u;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    double before = carry, total = carry;
#pragma unroll
    for (int w = 0; w < kPrepSmall / 32; ++w) {
      const double x = wsum[w];
      if (w < warp) before += x;
      total += x;
    }
    before += incl - v;  // the threads before this one in its warp
#pragma unroll
    for (int j = 0; j < kPrepRun; ++j) {
      if (tb + j < p.L) {
        p.beta[unit * p.L + tb + j] = d[j];
        p.cum[unit * p.L + tb + j] = before + run[j];
      }
    }
    carry = total;
    __syncthreads();  // wsum is rewritten next round
  }
}

// The same tile on the tensor cores (bf16 inputs, state 128): one CTA of 128
// threads per (lower tile, group, batch); the launch's blocks past those run
// the pre-pass (one per (batch, head)), which does not depend on C . B^T, so
// that both take one launch.  The TMA brings the tile's 128 query
// rows of C and 128 key rows of B as two 64-state slabs each (128-byte
// swizzle; rows past the sequence end arrive as zeros); one thread issues the
// eight K = 16 steps of the 128 x 128 x 128 product into 128 TMEM columns
// (row t in lane t, key s in column s); each warp then reads its quarter of
// the lanes and writes those rows to the workspace.  Both waits are bounded;
// a wait that runs out leaves NaN rows in the tile, so the failure shows in
// alpha, and the CTA still frees its TMEM.
struct __align__(1024) CbSmem {
  uint8_t C[2][kTile * 128];  // [slab]: 128 rows x 64 bf16
  uint8_t B[2][kTile * 128];
  uint64_t full, done;
  uint32_t taddr;
};
constexpr long long kCbWaitLimit = 2000000000ll;  // cycles (about a second)

__global__ void __launch_bounds__(128)
    attn_cb_tc_kernel(const __grid_constant__ CUtensorMap mB,
                      const __grid_constant__ CUtensorMap mC, AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the mask pass may start now: its zero tiles need nothing from this
  // launch, and its other tiles wait for it to finish (griddepcontrol.wait)
  pdl_launch_dependents();
  const int64_t ncb = p.ntri * p.G * p.batch;
  if ((int64_t)blockIdx.x >= ncb) {
    prep_unit_small<__nv_bfloat16>(p, (int64_t)blockIdx.x - ncb);
    return;
  }
  CbSmem &s = *reinterpret_cast<CbSmem *>(smem_raw +
                                          ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t li = (int64_t)blockIdx.x % p.ntri, g = ((int64_t)blockIdx.x / p.ntri) % p.G,
                b = (int64_t)blockIdx.x / (p.ntri * p.G);
  int64_t qt = (int64_t)((sqrt(8.0 * (double)li + 1.0) - 1.0) / 2.0);
  while (qt * (qt + 1) / 2 > li) --qt;
  while ((qt + 1) * (qt + 2) / 2 <= li) ++qt;
  const int64_t kt = li - qt * (qt + 1) / 2;

  if (tid == 0) {
    mbar_init(&s.full, 1);
    mbar_init(&s.done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.taddr, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s.taddr;

  if (tid == 0) {
    const int gx = (int)(g * 128);
    mbar_expect_tx(&s.full, 4 * kTile * 128);
    tma_load_3d(s.C[0], &mC, &s.full, gx, (int)(qt * kTile), (int)b);
    tma_load_3d(s.C[1], &mC, &s.full, gx + 64, (int)(qt * kTile), (int)b);
    tma_load_3d(s.B[0], &mB, &s.full, gx, (int)(kt * kTile), (int)b);
    tma_load_3d(s.B[1], &mB, &s.full, gx + 64, (int)(kt * kTile), (int)b);
    if (mbar_wait(&s.full, 0, kCbWaitLimit)) {
      tc_fence_after();
      const uint32_t id = idesc_bf16_f32(128, 128, false, false);
      const uint64_t dC = smem_desc(smem_u32(s.C[0]), 16, 1024, kSwizzle128B);
      const uint64_t dB = smem_desc(smem_u32(s.B[0]), 16, 1024, kSwizzle128B);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        // K step kk: slab kk / 4, 32 bytes per step inside the slab
        const uint32_t ko = ((kk >> 2) * (kTile * 128) + (kk & 3) * 32) >> 4;
        mma_ss(tb, dC + ko, dB + ko, id, kk > 0);
      }
      mma_commit(&s.done);
    }
  }
  const bool got = mbar_wait(&s.done, 0, kCbWaitLimit);
  const bool all = __all_sync(0xffffffffu, got);
  tc_fence_after();
  float *row = p.cb + ((b * p.G + g) * p.ntri + li) * (int64_t)(kTile * kTile) +
               (int64_t)(32 * warp + lane) * kTile;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
#pragma unroll 1
  for (int c = 0; c < kTile; c += 16) {
    uint32_t r[16];
    if (all) {
      tmem_ld16(tb + lane_base + (uint32_t)c, r);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) r[j] = 0x7fc00000u;  // NaN
    }
#pragma unroll
    for (int j = 0; j < 16; j += 4)
      *reinterpret_cast<float4 *>(row + c + j) =
          make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                      __uint_as_float(r[j + 3]));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tb, 128);
}

// The mask pass: one CTA per (query tile, key tile, run of heads of one
// group, batch row), 256 threads with the same element ownership as the
// C . B^T pass.  A tile above the diagonal is zeros; otherwise the thread
// reads its 64 values of C . B^T (from L2) once and, per head, scales them
// by the decay factors and streams the rows out.
//
// The CTAs cost unequal time (a diagonal tile takes an exponential per
// element, a tile above it only zeros), and the grid runs several waves, so
// the linear block index lists them dearest first -- every diagonal tile,
// then every tile below it, then the zero tiles -- and the block scheduler,
// which starts blocks in index order, fills the last wave with cheap ones.
struct MaskItem {
  int64_t qt, kt, hg, b;
};
__device__ __forceinline__ MaskItem mask_item(int64_t r, int64_t ntile, int64_t nhg,
                                              int64_t batch) {
  const int64_t hb = nhg * batch;
  const int64_t nd = ntile * hb, nb = ntile * (ntile - 1) / 2 * hb;
  int cls = 2;  // 2 above (zeros), 0 diagonal, 1 below
  if (r >= nb) {
    r -= nb;
    cls = r >= nd ? 1 : 0;
    if (cls == 1) r -= nd;
  }
  const int64_t k = r / hb, j = r % hb;
  MaskItem m;
  m.hg = j % nhg;
  m.b = j / nhg;
  if (cls == 0) {
    m.qt = m.kt = k;
  } else {
    // the k-th tile strictly below the diagonal, row by row: qt (qt - 1) / 2 <= k
    int64_t qt = (int64_t)((1.0 + sqrt(1.0 + 8.0 * (double)k)) / 2.0);
    while (qt * (qt - 1) / 2 > k) --qt;
    while ((qt + 1) * qt / 2 <= k) ++qt;
    const int64_t kt = k - qt * (qt - 1) / 2;
    m.qt = cls == 1 ? qt : kt;  // the zero tiles are the mirror images
    m.kt = cls == 1 ? kt : qt;
  }
  return m;
}

__global__ void __launch_bounds__(256) attn_mask_kernel(AttnParams p) {
  __shared__ __align__(16) float colf[kHeadsPerCta][kTile];  // per key: exp2(cum_r - cum_s) beta_s
  __shared__ __align__(16) float betas[kHeadsPerCta][kTile];
  __shared__ __align__(16) float rowf[kHeadsPerCta][kTile][4];  // per query, key block
  __shared__ double cq[kHeadsPerCta][kTile], ck[kHeadsPerCta][kTile];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int64_t L = p.L, H = p.H;
  const int64_t ntile = (L + kTile - 1) / kTile;
  const MaskItem mi =
      mask_item(blockIdx.x, ntile, (H + p.heads_per_cta - 1) / p.heads_per_cta, p.batch);
  const int64_t qt = mi.qt, kt = mi.kt;
  const int64_t t0 = qt * kTile, s0 = kt * kTile;
  const int64_t b = mi.b;
  const int64_t h0 = mi.hg * p.heads_per_cta;
  const int nh = (int)(H - h0 < p.heads_per_cta ? H - h0 : p.heads_per_cta);
  const int64_t g = h0 / (H / p.G);

  // row i of this thread's 8 x 8 block of head h's tile
  auto store_row = [&](int64_t h, int i, const float (&v)[8]) {
    const int64_t t = t0 + 8 * ty + i;
    if (t >= L) return;
    float *row = p.alpha + ((b * H + h) * L + t) * L + s0;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int c = 64 * half + 4 * tx;
      if (s0 + c + 4 <= L && (L & 3) == 0) {
        st_stream4(reinterpret_cast<float4 *>(row + c),
                   make_float4(v[4 * half], v[4 * half + 1], v[4 * half + 2], v[4 * half + 3]));
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (s0 + c + j < L) row[c + j] = v[4 * half + j];
      }
    }
  };

  if (kt > qt) {  // above the diagonal: zeros
    const float zero[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int hh = 0; hh < nh; ++hh)
      for (int i = 0; i < 8; ++i) store_row(h0 + hh, i, zero);
    return;
  }
  // C . B^T and the running sums come from the launch before this one
  pdl_wait();
  // every head's factors first (threads 0..127: one key each; 128..255: one
  // query each), read straight from the running sums -- all of a thread's
  // loads issued before any is used; one barrier
  if (tid < kTile) {
    const int64_t tk = s0 + tid;
    const int rk = (tid | 31) < (int)(L - s0) ? (tid | 31) : (int)(L - s0 - 1);
    double ckt[kHeadsPerCta], crk[kHeadsPerCta];
    float bt[kHeadsPerCta];
#pragma unroll
    for (int hh = 0; hh < kHeadsPerCta; ++hh) {
      if (hh < nh) {
        const int64_t base = (b * H + h0 + hh) * L;
        ckt[hh] = tk < L ? p.cum[base + tk] : 0.0;
        bt[hh] = tk < L ? p.beta[base + tk] : 0.f;
        crk[hh] = p.cum[base + s0 + rk];
      }
    }
#pragma unroll
    for (int hh = 0; hh < kHeadsPerCta; ++hh) {
      if (hh < nh) {
        colf[hh][tid] = ex2((float)(crk[hh] - ckt[hh])) * bt[hh];
        ck[hh][tid] = ckt[hh];
        betas[hh][tid] = bt[hh];
      }
    }
  } else {
    const int q = tid - kTile;
    const int64_t tq = t0 + q;
    double cqt[kHeadsPerCta], crk[kHeadsPerCta][4];
#pragma unroll
    for (int hh = 0; hh < kHeadsPerCta; ++hh) {
      if (hh < nh) {
        const int64_t base = (b * H + h0 + hh) * L;
        cqt[hh] = tq < L ? p.cum[base + tq] : 0.0;
#pragma unroll
        for (int J = 0; J < 4; ++J) {
          const int rk = (32 * J + 31) < (int)(L - s0) ? 32 * J + 31 : (int)(L - s0 - 1);
          crk[hh][J] = p.cum[base + s0 + rk];
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < kHeadsPerCta; ++hh) {
      if (hh < nh) {
        cq[hh][q] = cqt[hh];
#pragma unroll
        for (int J = 0; J < 4; ++J) rowf[hh][q][J] = ex2((float)(cqt[hh] - crk[hh][J]));
      }
    }
  }
  // The thread's 8 x 8 block of C . B^T in two halves of four rows (each
  // read from L2 once, the second after the first half's heads are done):
  // measured 3 % faster than the whole block at once at the same two CTAs
  // per SM; bounded to three CTAs per SM it spills and runs slower.
  const float *tile =
      p.cb + ((b * p.G + g) * p.ntri + lower_index(qt, kt)) * (int64_t)(kTile * kTile);
  float acc[4][8];
  auto load_half = [&](int hf) {
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const float *row = tile + (8 * ty + 4 * hf + ii) * kTile;
      const float4 u0 = *reinterpret_cast<const float4 *>(row + 4 * tx);
      const float4 u1 = *reinterpret_cast<const float4 *>(row + 64 + 4 * tx);
      acc[ii][0] = u0.x; acc[ii][1] = u0.y; acc[ii][2] = u0.z; acc[ii][3] = u0.w;
      acc[ii][4] = u1.x; acc[ii][5] = u1.y; acc[ii][6] = u1.z; acc[ii][7] = u1.w;
    }
  };
  load_half(0);
  __syncthreads();

  const bool diag = qt == kt;
#pragma unroll 1
  for (int hf = 0; hf < 2; ++hf) {
  if (hf == 1) load_half(1);
  for (int hh = 0; hh < nh; ++hh) {
    const int64_t h = h0 + hh;
    if (!diag) {
      // below the diagonal tile: every factor is rowf * colf (one key block
      // per column half of this thread)
      const float4 c0 = *reinterpret_cast<const float4 *>(&colf[hh][4 * tx]);
      const float4 c1 = *reinterpret_cast<const float4 *>(&colf[hh][64 + 4 * tx]);
      const float cf[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const int J0 = tx >> 3, J1 = 2 + (tx >> 3);
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int i = 4 * hf + ii;
        const int qi = 8 * ty + i;
        const float r0 = rowf[hh][qi][J0], r1 = rowf[hh][qi][J1];
        float v[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = acc[ii][j] * (r0 * cf[j]);
#pragma unroll
        for (int j = 4; j < 8; ++j) v[j] = acc[ii][j] * (r1 * cf[j]);
        store_row(h, i, v);
      }
    } else {
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int i = 4 * hf + ii;
        const int qi = 8 * ty + i;
        const int64_t tq = t0 + qi;
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int kj = (j < 4 ? 4 * tx : 60 + 4 * tx) + j;  // 4 tx + j, or 64 + 4 tx + (j - 4)
          const int64_t tk = s0 + kj;
          float f;
          if (tk > tq) {
            f = 0.f;
          } else if ((tq >> 5) > (tk >> 5)) {
            f = rowf[hh][qi][kj >> 5] * colf[hh][kj];  // below the diagonal 32 x 32 blocks
          } else {
            f = ex2((float)(cq[hh][qi] - ck[hh][kj])) * betas[hh][kj];  // on a diagonal block
          }
          v[j] = acc[ii][j] * f;
        }
        store_row(h, i, v);
      }
    }
  }
  }
}

template <typename T>
cudaError_t launch_t(const AttnParams &p, cudaStream_t s) {
  const int64_t units = p.batch * p.H;
  cudaError_t e;
  if (std::is_same<T, __nv_bfloat16>::value && p.N == 128) {
    // tensor-core C . B^T: B and C as [batch, L, G * 128] bf16, 64 x 128 boxes
    const uint64_t GN = (uint64_t)(p.G * 128);
    uint64_t dims[3] = {GN, (uint64_t)p.L, (uint64_t)p.batch};
    uint64_t strides[2] = {GN * 2, (uint64_t)p.L * GN * 2};
    uint32_t box[3] = {64, (uint32_t)kTile, 1};
    CUtensorMap mB, mC;
    if (!encode_tiled(&mB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.B, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tiled(&mC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.Cm, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const size_t smem = sizeof(CbSmem) + 1024;
    // (set on every call: the attribute belongs to the current device)
    const cudaError_t attr = cudaFuncSetAttribute(
        attn_cb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr != cudaSuccess) return attr;
    // C . B^T blocks first (the longer ones), then the pre-pass blocks
    attn_cb_tc_kernel<<<(unsigned)(p.ntri * p.G * p.batch + units), 128, smem, s>>>(mB, mC, p);
  } else {
    attn_prep_kernel<T><<<(unsigned)units, kPrep, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_cb_kernel<T><<<dim3((unsigned)(16 * p.ntri), (unsigned)p.G, (unsigned)p.batch), 256, 0,
                        s>>>(p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t ntile = (p.L + kTile - 1) / kTile;
  const int64_t nblocks =
      ntile * ntile * ((p.H + p.heads_per_cta - 1) / p.heads_per_cta) * p.batch;
  // a programmatic dependent of the launch before it, so that its zero
  // tiles are written while that launch still runs
  return launch_dependent(attn_mask_kernel, dim3((unsigned)nblocks), dim3(256), 0, s, p);
}

}  // namespace

// Heads per CTA: the largest divisor of heads-per-group not above four, so
// that a CTA's heads share one C . B^T.
int attn_heads_per_cta(int64_t H, int64_t G) {
  const int64_t hpg = H / G;
  for (int k = kHeadsPerCta; k > 1; --k)
    if (hpg % k == 0) return k;
  return 1;
}

bool attention_supported(const AttnParams &p) {
  const int64_t ntile = (p.L + kTile - 1) / kTile;
  const int64_t nhg = (p.H + p.heads_per_cta - 1) / p.heads_per_cta;
  const int64_t ntri = ntile * (ntile + 1) / 2;
  return p.N >= 1 && p.N <= 256 && ntile * ntile * nhg * p.batch < (1ll << 31) &&
         ntri * p.G * p.batch + p.batch * p.H < (1ll << 31) &&
         16 * (ntile * (ntile + 1) / 2) < (1ll << 31) && p.batch <= 65535 &&
         p.G <= 65535 && (p.H + p.heads_per_cta - 1) / p.heads_per_cta <= 65535;
}

// The steps and running sums (float64) per (batch, head, token), then C . B^T
// of every tile on or below the diagonal per (batch, group).
size_t attention_workspace_bytes(int64_t batch, int64_t H, int64_t G, int64_t L) {
  const int64_t ntile = (L + kTile - 1) / kTile;
  const int64_t ntri = ntile * (ntile + 1) / 2;
  return (((size_t)(batch * H * L) * (sizeof(double) + sizeof(float)) + 15) & ~(size_t)15) +
         (size_t)(batch * G * ntri) * kTile * kTile * sizeof(float);
}

int64_t attention_lower_tiles(int64_t L) {
  const int64_t ntile = (L + kTile - 1) / kTile;
  return ntile * (ntile + 1) / 2;
}

cudaError_t launch_attention(const AttnParams &p, cudaStream_t s) {
  return p.io == 1 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace ssm
