// ssd_tc.cu -- Mamba-2 SSD chunk scan on the sm_100a tensor cores (set b).
//
// What it computes ("Mamba-2", nnterp encyclopedia, "The hidden attention"
// and "The state"): per (batch, head), with step d_t = softplus(dt + bias),
// log-decay l_t = d_t A_h and, inside a tile of tokens, the inclusive sum
// cum_i of l,
//
//   y_i  = sum_{j<=i} (C_i . B_j) exp(cum_i - cum_j) d_j x_j       (masked form)
//        + exp(cum_i) C_i . h_prev                                  (carried state)
//        + D x_i,                        then * silu(z_i) if gated,
//   h    = exp(cum_last) h_prev + sum_j exp(cum_last - cum_j) d_j B_j x_j^T.
//
// The tile is 128 tokens, one TMEM lane per token, so a 256-token chunk is
// two tiles with the state carried between them -- the same arithmetic as the
// 256-token masked form, up to rounding.
//
// One CTA per (batch, head), warp-specialised, tiles pipelined:
//   warp 8      TMA producer: C, B ([128 x 128] bf16, two 64-column slabs) and
//               x ([128 x 64]), 128-byte swizzle, double-buffered stages.
//   warp 9      MMA issuer (tcgen05, bf16 in, fp32 accumulators in TMEM):
//                 S  = C B^T            A, B K-major          (two buffers)
//                 Yd = (S o mask) x     A = masked S from TMEM, B MN-major
//                 Sc = B^T (w o x)      A = B read MN-major, B = scaled x
//                 Yo = C h_prev         B = bf16 copy of the carried state
//               issued per tile in the order Sc(c), S(c+1), Yo(c), Yd(c).
//   warps 4-7   mask group, thread = token: the tile's step, cumulative decay
//               and weights, w o x, then the mask applied to S as it is read
//               from TMEM, written back as the bf16 A operand.  The mask
//               exp(cum_i - cum_j) d_j is elementwise only on the four 32 x 32
//               diagonal blocks; below them it is a row factor times a column
//               factor, both <= 1 for a decaying state.
//   warps 0-3   state group: thread n keeps row n of the float32 state in
//               registers, h = exp(cum_last) h + Sc, writes its bf16 copy for
//               the next tile's Yo; then, thread = token, the output
//               y = Yd + exp(cum_i) Yo + D x (* silu(z)).
// The carried-state chain per tile is only the state group's update; the
// contractions of the next tile run under it.
//
// Every wait is bounded.  A group votes on its waits (bar.red.or) so its
// threads always take the same branch; a wait that runs out sets the device
// status word and a shared abort flag, every role leaves its loop, and the
// CTA frees its TMEM and returns.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma.h"

namespace ssm {
namespace {

using namespace sm100;

constexpr int kQ = 128;   // tokens per tile
constexpr int kN = 128;   // state size
constexpr int kP = 64;    // head dim
constexpr int kThreads = 320;
constexpr long long kWaitLimit = 2000000000ll;  // cycles (about a second)

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColSc = 256, kColYd = 320, kColYo = 384;

struct __align__(1024) SsdSmem {
  uint8_t C[2][2][kQ * 128];  // [stage][slab]
  uint8_t B[2][2][kQ * 128];
  uint8_t X[2][kQ * 128];     // [stage]
  uint8_t Xw[2][kQ * 128];    // [tile parity]: w o x
  uint8_t Hb[kN * 128];       // bf16 copy of the carried state, rows n
  float cum[2][kQ];           // [tile parity]
  float dd[2][kQ];
  float vd[2][kQ];
  float e[2][kQ];
  float a[2];
  float wsum[4];
  // Per-tile signals come in pairs indexed by tile parity, so a waiter would
  // have to fall two tiles behind to miss a phase; the stage dependencies
  // bound every role's lead to one tile.
  uint64_t full[2], empty[2], sdone[2];
  uint64_t scdone[2], yodone[2], yddone[2], xready[2], mready[2], stdone[2], yfree[2];
  uint32_t taddr;
  int abort;
};

struct SsdTcParams {
  int64_t batch, L, H, G;
  uint32_t flags;
  const __nv_bfloat16 *dt, *z;
  const float *A, *D, *dt_bias, *h0;
  __nv_bfloat16 *y;
  float *h_last;
  int *status;
};

__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// Named barrier for one 128-thread group (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void group_sync(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}
// Group barrier that also ORs a predicate over the group.
__device__ __forceinline__ bool group_any(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool aborted(const SsdSmem &s) {
  return *(volatile const int *)&s.abort != 0;
}
__device__ __forceinline__ void set_abort(SsdSmem &s, int *status, int code) {
  *(volatile int *)&s.abort = 1;
  if (status) atomicExch(status, code);
}

// A single-thread role's wait.
__device__ __forceinline__ bool wait1(SsdSmem &s, uint64_t *bar, uint32_t parity, int *status,
                                      int code) {
  if (aborted(s)) return false;
  if (mbar_wait(bar, parity, kWaitLimit)) return true;
  set_abort(s, status, code);
  return false;
}
// A 128-thread group's wait: every thread waits (bounded), then the group votes.
__device__ __forceinline__ bool waitg(SsdSmem &s, int gid, uint64_t *bar, uint32_t parity,
                                      int *status, int code) {
  bool ok = !aborted(s) && mbar_wait(bar, parity, kWaitLimit);
  const bool fail = group_any(gid, !ok);
  if (fail && (threadIdx.x & 127) == 0) set_abort(s, status, code);
  return !fail;
}

__global__ void __launch_bounds__(kThreads, 1)
    ssd_tc_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mB,
                  const __grid_constant__ CUtensorMap mC, const SsdTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  SsdSmem &s = *reinterpret_cast<SsdSmem *>(base);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t hd = blockIdx.x, b = blockIdx.y;
  const int64_t L = p.L, H = p.H;
  const int g = (int)(hd / (H / p.G));
  const int nch = (int)((L + kQ - 1) / kQ);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 2);   // the tile's last MMA commit + the output group
      mbar_init(&s.sdone[i], 1);
      mbar_init(&s.scdone[i], 1);
      mbar_init(&s.yodone[i], 1);
      mbar_init(&s.yddone[i], 1);
      mbar_init(&s.xready[i], 1);
      mbar_init(&s.mready[i], 1);
      mbar_init(&s.stdone[i], 1);
      mbar_init(&s.yfree[i], 1);
    }
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&s.taddr, kTmemCols);
    tmem_relinquish();
  }

  // State group: row n of the carried state in float32 registers.
  float h[kP];
  if (warp < 4) {
    const float *src = p.h0 ? p.h0 + ((b * H + hd) * kN + tid) * kP : nullptr;
#pragma unroll
    for (int q = 0; q < kP; q += 4) {
      float4 v = src ? *reinterpret_cast<const float4 *>(src + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      h[q] = v.x; h[q + 1] = v.y; h[q + 2] = v.z; h[q + 3] = v.w;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float f[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) f[k] = h[8 * c + k];
      *reinterpret_cast<uint4 *>(s.Hb + sw128(tid, c)) = pack8(f);
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s.taddr;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&mX);
      tma_prefetch_desc(&mB);
      tma_prefetch_desc(&mC);
      for (int c = 0; c < nch; ++c) {
        const int st = c & 1;
        if (c >= 2 && !wait1(s, &s.empty[st], ((c >> 1) + 1) & 1, p.status, 1)) break;
        mbar_expect_tx(&s.full[st], 5 * kQ * 128);
        tma_load_3d(s.C[st][0], &mC, &s.full[st], g * kN, c * kQ, (int)b);
        tma_load_3d(s.C[st][1], &mC, &s.full[st], g * kN + 64, c * kQ, (int)b);
        tma_load_3d(s.B[st][0], &mB, &s.full[st], g * kN, c * kQ, (int)b);
        tma_load_3d(s.B[st][1], &mB, &s.full[st], g * kN + 64, c * kQ, (int)b);
        tma_load_4d(s.X[st], &mX, &s.full[st], 0, (int)hd, c * kQ, (int)b);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_S = idesc_bf16_f32(128, 128, false, false);
      const uint32_t id_Y = idesc_bf16_f32(128, 64, false, true);
      const uint32_t id_Sc = idesc_bf16_f32(128, 64, true, true);
      auto mma_S = [&](int c) {  // S(c) = C B^T into S[c & 1]
        const int st = c & 1;
        const uint32_t c0 = smem_u32(s.C[st][0]), b0 = smem_u32(s.B[st][0]);
        const uint32_t dcol = st ? kColS1 : kColS0;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t ko = (k >> 2) * (kQ * 128) + (k & 3) * 32;
          mma_ss(tb + dcol, smem_desc(c0 + ko, 16, 1024, kSwizzle128B),
                 smem_desc(b0 + ko, 16, 1024, kSwizzle128B), id_S, k > 0);
        }
        mma_commit(&s.sdone[st]);
      };
      bool ok = wait1(s, &s.full[0], 0, p.status, 2);
      if (ok) mma_S(0);
      for (int c = 0; ok && c < nch; ++c) {
        const int st = c & 1, pv = (c + 1) & 1;  // pv: parity slot of tile c-1
        const uint32_t ph = (c >> 1) & 1, php = ((c - 1) >> 1) & 1;
        // Sc(c) = B^T (w o x): needs w o x, and the state group done with Sc(c-1)
        if (!wait1(s, &s.xready[st], ph, p.status, 3)) break;
        if (c > 0 && !wait1(s, &s.stdone[pv], php, p.status, 4)) break;
        tc_fence_after();
        {
          const uint32_t b0 = smem_u32(s.B[st][0]), xw = smem_u32(s.Xw[st]);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ss(tb + kColSc, smem_desc(b0 + k * 2048, kQ * 128, 1024, kSwizzle128B),
                   smem_desc(xw + k * 2048, kQ * 128, 1024, kSwizzle128B), id_Sc, k > 0);
          mma_commit(&s.scdone[st]);
        }
        // S(c+1), as soon as its tile has landed
        if (c + 1 < nch) {
          if (!wait1(s, &s.full[(c + 1) & 1], ((c + 1) >> 1) & 1, p.status, 5)) break;
          mma_S(c + 1);
        }
        // Yo(c) = C h_prev: needs the output group done with Yo/Yd of c-1
        if (c > 0 && !wait1(s, &s.yfree[pv], php, p.status, 6)) break;
        tc_fence_after();
        {
          const uint32_t c0 = smem_u32(s.C[st][0]), hb = smem_u32(s.Hb);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t ko = (k >> 2) * (kQ * 128) + (k & 3) * 32;
            mma_ss(tb + kColYo, smem_desc(c0 + ko, 16, 1024, kSwizzle128B),
                   smem_desc(hb + k * 2048, kN * 128, 1024, kSwizzle128B), id_Y, k > 0);
          }
          mma_commit(&s.yodone[st]);
        }
        // Yd(c) = M x: needs the masked S
        if (!wait1(s, &s.mready[st], ph, p.status, 7)) break;
        tc_fence_after();
        {
          const uint32_t x0 = smem_u32(s.X[st]);
          const uint32_t mcol = st ? kColS1 : kColS0;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ts(tb + kColYd, tb + mcol + 8 * k,
                   smem_desc(x0 + k * 2048, kQ * 128, 1024, kSwizzle128B), id_Y, k > 0);
          mma_commit(&s.yddone[st]);
          mma_commit(&s.empty[st]);
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ mask group
    const int i = tid - 128;  // token of the tile; TMEM lane i
    const int mw = warp - 4;
    const uint32_t lane_base = (uint32_t)(32 * mw) << 16;
    const float A2 = p.A[hd] * kLog2e;
    const float bias = p.dt_bias ? p.dt_bias[hd] : 0.f;
    const bool softplus_on = p.flags & 1u;
    float dt_next = i < L ? ld(p.dt + (b * L + i) * H + hd) : 0.f;
    for (int c = 0; c < nch; ++c) {
      const int st = c & 1, k = c & 1;
      const int64_t t0 = (int64_t)c * kQ;
      const int valid = (int)(L - t0 < kQ ? L - t0 : kQ);
      if (!waitg(s, 1, &s.full[st], (c >> 1) & 1, p.status, 8)) break;
      // step, log2-decay and its inclusive sum over the tile
      float d = 0.f;
      if (i < valid) {
        d = dt_next + bias;
        if (softplus_on) d = softplus(d);
      }
      if (t0 + kQ + i < L) dt_next = ld(p.dt + (b * L + t0 + kQ + i) * H + hd);
      float cs = d * A2;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, cs, off);
        if (lane >= off) cs += v;
      }
      if (lane == 31) s.wsum[mw] = cs;
      group_sync(1);
      float total = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float v = s.wsum[w];
        if (w < mw) cs += v;
        total += v;
      }
      s.cum[k][i] = cs;
      s.dd[k][i] = d;
      s.e[k][i] = ex2(cs);
      if (i == 0) s.a[k] = ex2(total);
      group_sync(1);
      s.vd[k][i] = ex2(s.cum[k][mw * 32 + 31] - cs) * d;
      const float w_i = ex2(total - cs) * d;
      // w o x (row i), the B operand of Sc
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        float f[8];
        unpack8(*reinterpret_cast<const uint4 *>(s.X[st] + sw128(i, cc)), f);
#pragma unroll
        for (int q = 0; q < 8; ++q) f[q] *= w_i;
        *reinterpret_cast<uint4 *>(s.Xw[k] + sw128(i, cc)) = pack8(f);
      }
      fence_async_smem();
      group_sync(1);
      if (i == 0) mbar_arrive(&s.xready[k]);
      // masked S -> bf16 A operand, written over S as S is read
      if (!waitg(s, 1, &s.sdone[k], (c >> 1) & 1, p.status, 9)) break;
      tc_fence_after();
      {
        const uint32_t col = k ? kColS1 : kColS0;
        const float *cum = s.cum[k];
#pragma unroll
        for (int J = 0; J < 4; ++J) {
          uint32_t m[16];
          if (J > mw) {
#pragma unroll
            for (int q = 0; q < 16; ++q) m[q] = 0u;
          } else {
            uint32_t r0[16], r1[16];
            tmem_ld16(tb + lane_base + col + 32 * J, r0);
            tmem_ld16(tb + lane_base + col + 32 * J + 16, r1);
            tmem_ld_wait();
            float f[32];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              f[q] = __uint_as_float(r0[q]);
              f[16 + q] = __uint_as_float(r1[q]);
            }
            if (J < mw) {
              const float u = ex2(cs - cum[32 * J + 31]);
              const float *vd = s.vd[k] + 32 * J;
#pragma unroll
              for (int q = 0; q < 32; ++q) f[q] *= u * vd[q];
            } else {
              const float *dd = s.dd[k] + 32 * J;
#pragma unroll
              for (int q = 0; q < 32; ++q) {
                const int j = 32 * J + q;
                f[q] = (j <= i) ? f[q] * ex2(cs - cum[j]) * dd[q] : 0.f;
              }
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) m[q] = pack_bf16x2(f[2 * q], f[2 * q + 1]);
          }
          tmem_st16(tb + lane_base + col + 16 * J, m);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      group_sync(1);
      if (i == 0) mbar_arrive(&s.mready[k]);
    }
  } else {
    // ------------------------------------------------------------ state group
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const float Dh = p.D ? p.D[hd] : 0.f;
    for (int c = 0; c < nch; ++c) {
      const int st = c & 1, k = c & 1;
      const uint32_t ph = (c >> 1) & 1;
      const int64_t t0 = (int64_t)c * kQ;
      const int valid = (int)(L - t0 < kQ ? L - t0 : kQ);
      // h = a h + Sc (thread = row n); a and e come from the mask group
      if (!waitg(s, 2, &s.xready[k], ph, p.status, 10)) break;
      if (!waitg(s, 2, &s.scdone[k], ph, p.status, 11)) break;
      tc_fence_after();
      const float a_c = s.a[k];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t r[16];
        tmem_ld16(tb + lane_base + kColSc + 16 * q, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) h[16 * q + j] = fmaf(a_c, h[16 * q + j], __uint_as_float(r[j]));
      }
      // the bf16 copy for Yo(c+1), once Yo(c) has read the old one
      if (!waitg(s, 2, &s.yodone[k], ph, p.status, 12)) break;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        float f[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = h[8 * cc + j];
        *reinterpret_cast<uint4 *>(s.Hb + sw128(tid, cc)) = pack8(f);
      }
      fence_async_smem();
      tc_fence_before();
      group_sync(2);
      if (tid == 0) mbar_arrive(&s.stdone[k]);
      // output y = Yd + e_i Yo + D x (thread = token i)
      if (!waitg(s, 2, &s.yddone[k], ph, p.status, 13)) break;
      tc_fence_after();
      {
        const int i = tid;
        const float e_i = s.e[k][i];
        const int64_t row = (b * L + t0 + i) * H + hd;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t yd[16], yo[16];
          tmem_ld16(tb + lane_base + kColYd + 16 * q, yd);
          tmem_ld16(tb + lane_base + kColYo + 16 * q, yo);
          tmem_ld_wait();
          float x0[8], x1[8], o[16];
          unpack8(*reinterpret_cast<const uint4 *>(s.X[st] + sw128(i, 2 * q)), x0);
          unpack8(*reinterpret_cast<const uint4 *>(s.X[st] + sw128(i, 2 * q + 1)), x1);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float xv = j < 8 ? x0[j] : x1[j - 8];
            o[j] = fmaf(e_i, __uint_as_float(yo[j]), __uint_as_float(yd[j])) + Dh * xv;
          }
          if (i < valid) {
            if (p.z) {
              const uint4 *zp = reinterpret_cast<const uint4 *>(p.z + row * kP + 16 * q);
              float z0[8], z1[8];
              unpack8(zp[0], z0);
              unpack8(zp[1], z1);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                o[j] *= silu(z0[j]);
                o[8 + j] *= silu(z1[j]);
              }
            }
            float lo[8], hi[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              lo[j] = o[j];
              hi[j] = o[8 + j];
            }
            uint4 *yp = reinterpret_cast<uint4 *>(p.y + row * kP + 16 * q);
            yp[0] = pack8(lo);
            yp[1] = pack8(hi);
          }
        }
      }
      tc_fence_before();
      group_sync(2);
      if (tid == 0) {
        mbar_arrive(&s.yfree[k]);
        mbar_arrive(&s.empty[st]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp < 4 && !aborted(s) && p.h_last) {
    float *dst = p.h_last + ((b * H + hd) * kN + tid) * kP;
#pragma unroll
    for (int q = 0; q < kP; q += 4)
      *reinterpret_cast<float4 *>(dst + q) = make_float4(h[q], h[q + 1], h[q + 2], h[q + 3]);
  }
  if (warp == 9) tmem_dealloc(tb, kTmemCols);
}

bool encode(CUtensorMap *m, const void *ptr, int rank, const uint64_t *dims,
            const uint64_t *strides, const uint32_t *box) {
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, ptr, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool ssd_tc_supported(const M2Params &p) {
  return p.io == 1 && p.N == kN && p.P == kP && p.states == nullptr && p.H <= 65535 &&
         p.L < (1ll << 31) && p.batch <= 65535;
}

size_t ssd_tc_smem_bytes() { return sizeof(SsdSmem) + 1024; }

cudaError_t launch_ssd_tc(const M2Params &p, int *status, cudaStream_t stream) {
  const int64_t GN = p.G * kN;
  CUtensorMap mX, mB, mC;
  {
    uint64_t dims[4] = {(uint64_t)kP, (uint64_t)p.H, (uint64_t)p.L, (uint64_t)p.batch};
    uint64_t strides[3] = {(uint64_t)kP * 2, (uint64_t)(p.H * kP * 2),
                           (uint64_t)(p.L * p.H * kP * 2)};
    uint32_t box[4] = {64, 1, kQ, 1};
    if (!encode(&mX, p.x, 4, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[3] = {(uint64_t)GN, (uint64_t)p.L, (uint64_t)p.batch};
    uint64_t strides[2] = {(uint64_t)GN * 2, (uint64_t)(p.L * GN * 2)};
    uint32_t box[3] = {64, kQ, 1};
    if (!encode(&mB, p.B, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!encode(&mC, p.Cm, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  SsdTcParams q;
  q.batch = p.batch;
  q.L = p.L;
  q.H = p.H;
  q.G = p.G;
  q.flags = p.flags;
  q.dt = static_cast<const __nv_bfloat16 *>(p.dt);
  q.z = static_cast<const __nv_bfloat16 *>(p.z);
  q.A = p.A;
  q.D = p.D;
  q.dt_bias = p.dt_bias;
  q.h0 = p.h0;
  q.y = static_cast<__nv_bfloat16 *>(p.y);
  q.h_last = p.h_last;
  q.status = status;
  const size_t smem = ssd_tc_smem_bytes();
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(ssd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((unsigned)p.H, (unsigned)p.batch);
  ssd_tc_kernel<<<grid, kThreads, smem, stream>>>(mX, mB, mC, q);
  return cudaGetLastError();
}

}  // namespace ssm
