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
// One CTA (4 warps, 128 threads) owns one (batch, head) and walks the tiles in
// order; two CTAs share an SM (256 TMEM columns and ~100 KB of shared memory
// each), so one's tensor-core work overlaps the other's elementwise work.
// Per tile, TMA brings C and B ([128 x 128] bf16, two 64-column slabs,
// 128-byte swizzle) and x ([128 x 64]); the next tile's C is fetched as soon
// as this tile's MMAs on C finish, B and x as soon as the state MMA
// finishes.  Four tcgen05 MMAs (bf16 in, fp32 accumulate in TMEM) do the
// contractions:
//   S   = C B^T                 [128 x 128]   A, B K-major from shared memory
//   Yd  = (S o mask) x          [128 x 64]    A = masked S, bf16, from TMEM
//   Sc  = B^T (w o x)           [128 x 64]    A = B read MN-major, B = x scaled
//                                             in place once the output is out
//   Yo  = C h_prev              [128 x 64]    B = bf16 copy of the carried state
// The mask exp(cum_i - cum_j) d_j is applied elementwise only on the four
// 32 x 32 diagonal blocks; below them it factors as
// exp(cum_i - cum_r) * exp(cum_r - cum_j) d_j with r the last token of the
// column block, both factors <= 1 for a decaying state.  The carried state
// stays in float32 registers (thread n holds row n); only its copy used as
// an MMA operand is rounded to bf16.
//
// Every wait is bounded; a wait that runs out sets the device status word, and
// the CTA stops issuing work, frees its TMEM and returns.
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
constexpr long long kWaitLimit = 2000000000ll;  // cycles (about a second)

// TMEM columns (256 per CTA, so two CTAs share an SM): the masked S is
// written over S as it is read, and the tile's state contribution reuses the
// half of S that is dead by then.
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColM = 0, kColSc = 64, kColYd = 128, kColYo = 192;

struct __align__(1024) SsdSmem {
  uint8_t C[2][kQ * 128];  // [slab]: 128 tokens x 64 state values, 128-byte swizzle
  uint8_t B[2][kQ * 128];
  uint8_t X[kQ * 128];     // 128 tokens x 64 head values; later w o x in place
  uint8_t Hb[kN * 128];    // bf16 copy of the carried state, rows n
  float cum[kQ];
  float dd[kQ];
  float vd[kQ];
  float wsum[4];
  uint64_t full_c, full_bx, bar_s, bar_y, bar_sc;
  uint32_t taddr;
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

// Every thread waits with a bound, then the CTA votes, so all threads take
// the same branch: either every wait completed, or the CTA records the
// failure in the status word and stops.
__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity, int *status, int code) {
  const bool ok = mbar_wait(bar, parity, kWaitLimit);
  const bool any_fail = __syncthreads_or(!ok) != 0;
  if (any_fail && threadIdx.x == 0 && status) atomicExch(status, code);
  return !any_fail;
}

__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

__global__ void __launch_bounds__(128, 2)
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
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  const float A2 = p.A[hd] * kLog2e;
  const float bias = p.dt_bias ? p.dt_bias[hd] : 0.f;
  const float Dh = p.D ? p.D[hd] : 0.f;
  const bool softplus_on = p.flags & 1u;

  if (tid == 0) {
    mbar_init(&s.full_c, 1);
    mbar_init(&s.full_bx, 1);
    mbar_init(&s.bar_s, 1);
    mbar_init(&s.bar_y, 1);
    mbar_init(&s.bar_sc, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mX);
    tma_prefetch_desc(&mB);
    tma_prefetch_desc(&mC);
  }
  if (warp == 0) {
    tmem_alloc(&s.taddr, kTmemCols);
    tmem_relinquish();
  }

  // Carried state: thread n holds row n (64 values) in float32.
  float h[kP];
  {
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
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s.taddr;

  auto load_c = [&](int c) {
    mbar_expect_tx(&s.full_c, 2 * kQ * 128);
    tma_load_3d(s.C[0], &mC, &s.full_c, g * kN, c * kQ, (int)b);
    tma_load_3d(s.C[1], &mC, &s.full_c, g * kN + 64, c * kQ, (int)b);
  };
  auto load_bx = [&](int c) {
    mbar_expect_tx(&s.full_bx, 3 * kQ * 128);
    tma_load_3d(s.B[0], &mB, &s.full_bx, g * kN, c * kQ, (int)b);
    tma_load_3d(s.B[1], &mB, &s.full_bx, g * kN + 64, c * kQ, (int)b);
    tma_load_4d(s.X, &mX, &s.full_bx, 0, (int)hd, c * kQ, (int)b);
  };
  if (tid == 0) {
    load_c(0);
    load_bx(0);
  }

  const uint32_t id_S = idesc_bf16_f32(128, 128, false, false);
  const uint32_t id_Y = idesc_bf16_f32(128, 64, false, true);
  const uint32_t id_Sc = idesc_bf16_f32(128, 64, true, true);

  // Raw step of this thread's token, one tile ahead.
  float dt_next = 0.f;
  if (tid < L) dt_next = ld(p.dt + (b * L + tid) * H + hd);

  bool aborted = false;
  for (int c = 0; c < nch; ++c) {
    const uint32_t par = c & 1;
    const int64_t t0 = (int64_t)c * kQ;
    const int valid = (int)(L - t0 < kQ ? L - t0 : kQ);

    // ---- step, log2-decay and its inclusive sum over the tile (thread = token)
    float d = 0.f;
    if (tid < valid) {
      d = dt_next + bias;
      if (softplus_on) d = softplus(d);
    }
    if (t0 + kQ + tid < L) dt_next = ld(p.dt + (b * L + t0 + kQ + tid) * H + hd);
    float cs = d * A2;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float v = __shfl_up_sync(0xffffffffu, cs, off);
      if (lane >= off) cs += v;
    }
    if (lane == 31) s.wsum[warp] = cs;
    __syncthreads();
    float total = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float v = s.wsum[w];
      if (w < warp) cs += v;
      total += v;
    }
    s.cum[tid] = cs;
    s.dd[tid] = d;
    __syncthreads();
    // v_j = exp2(cum_r - cum_j) d_j with r the last token of j's 32-block
    s.vd[tid] = ex2(s.cum[warp * 32 + 31] - cs) * d;
    const float e_i = ex2(cs);                 // decay of the carried state to token i
    const float w_i = ex2(total - cs) * d;     // weight of token i in the tile's state
    const float a_c = ex2(total);              // decay across the whole tile

    // ---- S = C B^T and Yo = C h_prev
    {
      const bool ok_c = mbar_wait(&s.full_c, par, kWaitLimit);
      const bool ok_bx = mbar_wait(&s.full_bx, par, kWaitLimit);
      if (__syncthreads_or(!(ok_c && ok_bx))) {
        if (tid == 0 && p.status) atomicExch(p.status, 1);
        aborted = true;
        break;
      }
    }
    if (tid == 0) {
      tc_fence_after();
      const uint32_t c0 = smem_u32(s.C[0]), b0 = smem_u32(s.B[0]), hb = smem_u32(s.Hb);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t ko = (k >> 2) * (kQ * 128) + (k & 3) * 32;
        mma_ss(tb + kColS, smem_desc(c0 + ko, 16, 1024, kSwizzle128B),
               smem_desc(b0 + ko, 16, 1024, kSwizzle128B), id_S, k > 0);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t ko = (k >> 2) * (kQ * 128) + (k & 3) * 32;
        mma_ss(tb + kColYo, smem_desc(c0 + ko, 16, 1024, kSwizzle128B),
               smem_desc(hb + k * 2048, kN * 128, 1024, kSwizzle128B), id_Y, k > 0);
      }
      mma_commit(&s.bar_s);
    }
    if (!wait_all(&s.bar_s, par, p.status, 2)) { aborted = true; break; }
    tc_fence_after();
    // C is free: fetch the next tile's C under the rest of this tile.
    if (tid == 0 && c + 1 < nch) load_c(c + 1);

    // ---- masked S -> bf16 A operand in TMEM, written over S as S is read
    {
      const float cum_i = cs;
#pragma unroll
      for (int J = 0; J < 4; ++J) {
        uint32_t m[16];
        if (J > warp) {
#pragma unroll
          for (int k = 0; k < 16; ++k) m[k] = 0u;
        } else {
          uint32_t r0[16], r1[16];
          tmem_ld16(tb + lane_base + kColS + 32 * J, r0);
          tmem_ld16(tb + lane_base + kColS + 32 * J + 16, r1);
          tmem_ld_wait();
          float f[32];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            f[k] = __uint_as_float(r0[k]);
            f[16 + k] = __uint_as_float(r1[k]);
          }
          if (J < warp) {
            const float u = ex2(cum_i - s.cum[32 * J + 31]);
#pragma unroll
            for (int k = 0; k < 32; ++k) f[k] *= u * s.vd[32 * J + k];
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const int j = 32 * J + k;
              f[k] = (j <= tid) ? f[k] * ex2(cum_i - s.cum[j]) * s.dd[j] : 0.f;
            }
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) m[k] = pack_bf16x2(f[2 * k], f[2 * k + 1]);
        }
        tmem_st16(tb + lane_base + kColM + 16 * J, m);
      }
      tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t x0 = smem_u32(s.X);
#pragma unroll
      for (int k = 0; k < 8; ++k)  // Yd = M x
        mma_ts(tb + kColYd, tb + kColM + 8 * k,
               smem_desc(x0 + k * 2048, kQ * 128, 1024, kSwizzle128B), id_Y, k > 0);
      mma_commit(&s.bar_y);
    }
    if (!wait_all(&s.bar_y, par, p.status, 3)) { aborted = true; break; }
    tc_fence_after();

    // ---- output y = Yd + e_i Yo + D x (thread i = token i), then w o x in place
    {
      const int64_t row = (b * L + t0 + tid) * H + hd;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t yd[16], yo[16];
        tmem_ld16(tb + lane_base + kColYd + 16 * q, yd);
        tmem_ld16(tb + lane_base + kColYo + 16 * q, yo);
        tmem_ld_wait();
        uint4 *xp0 = reinterpret_cast<uint4 *>(s.X + sw128(tid, 2 * q));
        uint4 *xp1 = reinterpret_cast<uint4 *>(s.X + sw128(tid, 2 * q + 1));
        float x0[8], x1[8], o[16];
        unpack8(*xp0, x0);
        unpack8(*xp1, x1);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float xv = k < 8 ? x0[k] : x1[k - 8];
          o[k] = fmaf(e_i, __uint_as_float(yo[k]), __uint_as_float(yd[k])) + Dh * xv;
        }
        if (tid < valid) {
          if (p.z) {
            const uint4 *zp = reinterpret_cast<const uint4 *>(p.z + row * kP + 16 * q);
            float z0[8], z1[8];
            unpack8(zp[0], z0);
            unpack8(zp[1], z1);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              o[k] *= silu(z0[k]);
              o[8 + k] *= silu(z1[k]);
            }
          }
          float a[8], bb[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            a[k] = o[k];
            bb[k] = o[8 + k];
          }
          uint4 *yp = reinterpret_cast<uint4 *>(p.y + row * kP + 16 * q);
          yp[0] = pack8(a);
          yp[1] = pack8(bb);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          x0[k] *= w_i;
          x1[k] *= w_i;
        }
        *xp0 = pack8(x0);
        *xp1 = pack8(x1);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t b0 = smem_u32(s.B[0]), xw = smem_u32(s.X);
#pragma unroll
      for (int k = 0; k < 8; ++k)  // Sc = B^T (w o x)
        mma_ss(tb + kColSc, smem_desc(b0 + k * 2048, kQ * 128, 1024, kSwizzle128B),
               smem_desc(xw + k * 2048, kQ * 128, 1024, kSwizzle128B), id_Sc, k > 0);
      mma_commit(&s.bar_sc);
    }
    if (!wait_all(&s.bar_sc, par, p.status, 4)) { aborted = true; break; }
    tc_fence_after();
    // B and x are free: fetch the next tile's.
    if (tid == 0 && c + 1 < nch) load_bx(c + 1);

    // ---- carried state: h = a h + Sc  (thread n = row n)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t r[16];
      tmem_ld16(tb + lane_base + kColSc + 16 * q, r);
      tmem_ld_wait();
#pragma unroll
      for (int k = 0; k < 16; ++k) h[16 * q + k] = fmaf(a_c, h[16 * q + k], __uint_as_float(r[k]));
    }
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      float f[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) f[k] = h[8 * cc + k];
      *reinterpret_cast<uint4 *>(s.Hb + sw128(tid, cc)) = pack8(f);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (!aborted && p.h_last) {
    float *dst = p.h_last + ((b * H + hd) * kN + tid) * kP;
#pragma unroll
    for (int q = 0; q < kP; q += 4)
      *reinterpret_cast<float4 *>(dst + q) = make_float4(h[q], h[q + 1], h[q + 2], h[q + 3]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tb, kTmemCols);
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
  ssd_tc_kernel<<<grid, 128, smem, stream>>>(mX, mB, mC, q);
  return cudaGetLastError();
}

}  // namespace ssm
