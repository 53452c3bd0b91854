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
//   warp 12     TMA producer: C, B ([128 x 128] bf16, two 64-column slabs) and
//               x ([128 x 64]), 128-byte swizzle, double-buffered stages.
//   warp 13     MMA issuer (tcgen05, bf16 in, fp32 accumulators in TMEM):
//                 S  = C B^T                 A, B K-major     (two buffers)
//                 Sc = B^T (w o x)           A = B read MN-major (two buffers)
//                 Y  = M x + (e o C) h_prev  A = M and e o C from TMEM, both
//                                            held in S's columns (two buffers)
//               per tile Sc(c) and S(c+1) in whichever order their inputs
//               arrive, then Y(c).
//   warps 4-7 and 14-17   mask group, thread = token, two warps per TMEM
//               lane quarter each taking half of every row's work (each warp
//               also recomputes the whole tile's decay factors, so the warps
//               run unsynchronised): the tile's steps d_j and decays
//               a_j = exp(d_j A), and every factor exp(cum_i - cum_j) as the
//               product a_{j+1} .. a_i (never as the exponential of a
//               difference of running sums, which would lose a small step
//               beside a large sum); it publishes the column factor w_j for
//               the output group; then the mask applied to S as it is read
//               from TMEM (D on its diagonal, so Y holds D x), and the
//               row-scaled C, e_i C_i with e_i = a_0 .. a_i, both written
//               back as the bf16 A operand of Y.  The mask is elementwise on
//               the four 32 x 32 diagonal blocks (a running product down from
//               the diagonal); below them it is a row factor times a column
//               factor, both <= 1 for a decaying state.
//   warps 0-3   state group: thread n keeps row n of the float32 state in
//               registers, h = exp(cum_last) h + Sc, and writes its bf16 copy
//               for Y of the next tile (two buffers).
//   warps 8-11  output group: w o x of the next tile (the B operand of Sc,
//               from the landed x and the mask group's w_j), then y = Y
//               (* silu(z)) of this tile, thread = token.  In the fused form
//               (the mixer's causal convolution in front, "Mamba-2", the
//               module tree and "The mixer's values": x, B, C =
//               silu(conv1d(xBC))), the same pass first convolves the landed
//               x tile in place: thread (4 channels, 16 tokens) walks its
//               tokens with the three previous raw inputs in registers, the
//               three rows before the tile kept from the previous tile.  The
//               mask group never reads x, so the convolution runs beside the
//               S product and the mask.  B and C, which every head of a
//               group shares, are convolved once by ssd_bc_conv_kernel
//               before the scan.
// With Y, Sc and the bf16 state double-buffered, the only chain carried from
// tile to tile is the state group's update; every other role has a tile of
// slack, and the contractions of the next tile run under this tile's
// elementwise work.  Signals: full/empty (stages), wready (w_j and the tile
// decay, mask -> output and state groups, four deep), xready (w o x, output
// -> MMA), sdone/scdone/yready (MMA commits), mready, stdone, yfree.
//
// A CTA runs either a whole (batch, head) unit or a segment of its tiles:
// when the last wave of units is partial, the host cuts those units into
// sequence segments (first every segment from its own start, then
// ssd_seg_carry_kernel chains the end states -- the state is linear in the
// start state, with one scalar decay per tile -- then the segments again
// from the carried states beside the whole units).
//
// Every wait is bounded and every warp votes on its waits, so its lanes
// always take the same branch; warps of a group never wait for each other,
// they arrive once per warp on four-count barriers.  A wait that runs out sets the
// device status word and a shared abort flag, every role leaves its loop, the
// MMA issuer and the producer wait (bounded) for their operations in flight,
// and the CTA frees its TMEM and returns.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma.h"

#include <algorithm>

namespace ssm {
namespace {

using namespace sm100;

constexpr int kQ = 128;   // tokens per tile
constexpr int kN = 128;   // state size
constexpr int kP = 64;    // head dim
constexpr int kThreads = 576;  // 18 warps; the fused form adds two (640)
template <bool CONV>
constexpr int threads_of() { return CONV ? kThreads + 64 : kThreads; }
constexpr long long kWaitLimit = 2000000000ll;  // cycles (about a second)

// TMEM columns: S[2] (fp32 S; then masked S in the first 64 columns and e o C
// in the next 64, as packed bf16), Sc[2], Y[2].
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColSc = 256, kColY = 384;

struct __align__(1024) SsdSmem {
  uint8_t C[2][2][kQ * 128];  // [stage][slab]
  uint8_t B[2][2][kQ * 128];
  uint8_t X[2][kQ * 128];     // [stage]
  uint8_t Xw[kQ * 128];       // w o x of the tile whose Sc is next
  uint8_t Hb[2][kN * 128];    // bf16 copy of the carried state, rows n
  float adw[8][kQ];           // per mask-group warp: decay a_j of token j,
  float ppw[8][kQ];           //   a_b ... a_j (b the first token of j's 32-token block),
  float ddw[8][kQ];           //   step d_j,
  float vdw[8][kQ];           //   a_{j+1} ... a_{b+31} d_j (column factor of the mask)
  // The column factor w_j of the tile's tokens (bf16, as the w o x product
  // uses it), from the mask group to the output group; four buffers, like
  // wready: the mask group may publish tile c + 2 before the output group
  // has read tile c (it need only wait for w o x of tile c - 1), but tile
  // c + 4 only after w o x of tile c + 1.
  __nv_bfloat16 wt[4][kQ];
  // With the convolution fused: the three raw inputs before a tile (bf16,
  // 64 channels).
  __nv_bfloat16 halo[3][kP];
  float a[4];                 // exp(cum_last) = a_0 .. a_127 per tile, ring of four
  // Per-tile signals come in pairs indexed by tile parity (wready in fours);
  // the dependencies between roles bound every waiter's lag to less than one
  // lap of its ring, so no waiter can miss a phase.
  uint64_t full[2], empty[2], sdone[2], scdone[2], mready[2], stdone[2], yready[2], yfree[2];
  uint64_t xready[2];         // w o x written (output group)
  uint64_t xconv[2];          // x convolved in place (convolution group, fused form)
  uint64_t wready[4];         // w_j and the tile decay written (mask group)
  uint32_t taddr;
  int abort;
};

// The CTA's dynamic shared memory (the struct plus 1 KB to align it) must
// fit the 227 KB a CTA may have.
static_assert(sizeof(SsdSmem) + 1024 <= 232448, "SsdSmem exceeds the shared memory of a CTA");

// Packed-bf16 TMEM columns (within an S buffer) of Y's A operand.  The mask
// for tokens 32 J + 16 h .. + 16 (K step 2 J + h of M x), written by the
// mask warp of half h, sits inside the S columns that warp itself read
// (its halves of fp32 blocks 0 and 1); e o C for states 16 kk .. + 16 (K
// step kk of (e o C) h_prev) sits inside the S columns the warp of half
// kk / 4 read in blocks 2 and 3.
__host__ __device__ constexpr uint32_t mask_col(int J, int h) {
  return 32u * (uint32_t)(J >> 1) + 16u * (uint32_t)h + 8u * (uint32_t)(J & 1);
}
__host__ __device__ constexpr uint32_t ec_col(int kk) {
  return 64u + 16u * (uint32_t)(kk >> 2) + 32u * (uint32_t)((kk >> 1) & 1) + 8u * (uint32_t)(kk & 1);
}

struct SsdTcParams {
  int64_t batch, L, H, G;
  uint32_t flags;
  const __nv_bfloat16 *dt, *z;
  const float *A, *D, *dt_bias, *h0;
  __nv_bfloat16 *y;
  float *h_last;
  int *status;
  // Work of a 1-D grid: blocks [0, nfull) run the whole (batch, head) units
  // 0 .. nfull - 1 (unit = b H + h); the others run segments seg_lo .. nseg - 1
  // of the tail units tail0 .. tail0 + ntail - 1, segment s covering tiles
  // [s nch / nseg, (s + 1) nch / nseg) of the sequence.
  int64_t nfull, tail0, ntail;
  int nseg, seg_lo;
  float *seg_hend;       // [ntail][nseg][N][P]: end state from the segment's own start state
  float *seg_decay;      // [ntail][nseg]: product of the segment's tile decays
  const float *seg_hin;  // [ntail][nseg][N][P]: the state entering each segment
  // The fused convolution (CONV): x is read from xBC before the convolution
  // (row stride ctot), convolved over tokens with the width-4 kernel cw
  // [ctot][4] and bias cbias, then silu; the inputs before token 0 come from
  // cs_in [batch][ctot][3] (oldest first) or are zeros.
  const __nv_bfloat16 *xbc;
  int64_t ctot;
  const float *cw, *cbias, *cs_in;
};

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One lane of the (fully active) warp is elected; the others get false.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// a * b on two packed bfloat16 pairs, round to nearest even.
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 16-byte global load / store that bypass L1 allocation (streamed once).
__device__ __forceinline__ uint4 ld_cs_u4(const void *p) {
  uint4 r;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ void st_cs_u4(void *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// Named barrier 1 over the convolution group of the fused form (warps 18
// and 19, 64 threads), and the same barrier as a vote: every thread of the
// group gets the OR of `v`.
constexpr int kConvThreads = 64;
__device__ __forceinline__ void conv_group_sync() { asm volatile("bar.sync 1, 64;" ::: "memory"); }
__device__ __forceinline__ bool conv_group_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, 64, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// 16-byte read-only global load.
__device__ __forceinline__ uint4 ld_nc_u4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void unpack8(uint4 u, float (&v)[8]) {
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
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
// A warp's wait: every lane polls (bounded), then the warp votes, so its
// lanes always take the same branch.  (Polling from lane 0 alone, with the
// verdict broadcast, measured slower.)
__device__ __forceinline__ bool waitw(SsdSmem &s, uint64_t *bar, uint32_t parity, int *status,
                                      int code) {
  // (no abort-flag read on this path: a role that gave up stops arriving,
  // and every wait on it runs out by itself)
  const bool ok = mbar_wait(bar, parity, kWaitLimit);
  const bool fail = __any_sync(0xffffffffu, !ok);
  if (fail && (threadIdx.x & 31) == 0) set_abort(s, status, code);
  return !fail;
}

template <bool CONV>
__global__ void __launch_bounds__(threads_of<CONV>(), 1)
    ssd_tc_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mB,
                  const __grid_constant__ CUtensorMap mC, const SsdTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  SsdSmem &s = *reinterpret_cast<SsdSmem *>(base);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t L = p.L, H = p.H;
  // The launch of whole units and carried segments is a programmatic
  // dependent of the carry: the whole units (first in block order) need
  // nothing from it and start at once; a carried segment waits for it.
  if (p.seg_lo > 0 && (int64_t)blockIdx.x >= p.nfull) pdl_wait();
  // This CTA's unit, its tiles [cb, cb + nch), where its start state comes
  // from and where its end state goes.  With seg_lo == 0 (the first pass over
  // the tail) a segment other than the first starts from zeros, writes no y
  // and leaves its end state and decay product for the carry; with seg_lo > 0
  // it starts from the carried state and writes y (and the last one h_last).
  const int nch_all = (int)((L + kQ - 1) / kQ);
  int64_t unit;
  int cb = 0, ce = nch_all;
  const float *h0u;
  float *hlu, *decu = nullptr;
  bool write_y = true;
  if ((int64_t)blockIdx.x < p.nfull) {
    unit = blockIdx.x;
    h0u = p.h0 ? p.h0 + unit * kN * kP : nullptr;
    hlu = p.h_last ? p.h_last + unit * kN * kP : nullptr;
  } else {
    const int per = p.nseg - p.seg_lo;
    const int64_t r = (int64_t)blockIdx.x - p.nfull;
    const int64_t tu = r / per;
    const int sg = p.seg_lo + (int)(r % per);
    const int64_t slot = tu * p.nseg + sg;
    unit = p.tail0 + tu;
    cb = (int)((int64_t)sg * nch_all / p.nseg);
    ce = (int)((int64_t)(sg + 1) * nch_all / p.nseg);
    if (p.seg_lo == 0) {
      h0u = (sg == 0 && p.h0) ? p.h0 + unit * kN * kP : nullptr;
      hlu = p.seg_hend + slot * kN * kP;
      decu = p.seg_decay + slot;
      write_y = sg == 0;
    } else {
      h0u = p.seg_hin + slot * kN * kP;
      hlu = (sg == p.nseg - 1 && p.h_last) ? p.h_last + unit * kN * kP : nullptr;
    }
  }
  const int64_t hd = unit % H, b = unit / H;
  const int g = (int)(hd / (H / p.G));
  const int nch = ce - cb;
  // TMEM lane quarter of this warp (warp i may only touch lanes 32 (i % 4) ..)
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
      mbar_init(&s.sdone[i], 1);
      mbar_init(&s.scdone[i], 1);
      mbar_init(&s.mready[i], 8);  // one arrival per mask-group warp
      mbar_init(&s.stdone[i], 4);  // one arrival per state-group warp
      mbar_init(&s.yready[i], 1);
      mbar_init(&s.yfree[i], 4);   // one arrival per output-group warp
    }
    for (int i = 0; i < 2; ++i) mbar_init(&s.xready[i], 4);  // one arrival per output warp
    for (int i = 0; i < 2; ++i) mbar_init(&s.xconv[i], 2);   // one per convolution warp
    for (int i = 0; i < 4; ++i) mbar_init(&s.wready[i], 4);  // one per half-0 mask warp
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(&s.taddr, kTmemCols);
    tmem_relinquish();
  }

  // The bf16 copy of the initial state, for Y(0), goes to Hb[1] (tile c
  // reads Hb[(c + 1) & 1]).
  if (warp < 4) {
    const float *src = h0u ? h0u + tid * kP : nullptr;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
      if (src) {
        v0 = *reinterpret_cast<const float4 *>(src + 8 * cc);
        v1 = *reinterpret_cast<const float4 *>(src + 8 * cc + 4);
      }
      *reinterpret_cast<uint4 *>(s.Hb[1] + sw128(tid, cc)) =
          make_uint4(pack_bf16x2(v0.x, v0.y), pack_bf16x2(v0.z, v0.w), pack_bf16x2(v1.x, v1.y),
                     pack_bf16x2(v1.z, v1.w));
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s.taddr;

  if (warp == 12) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&mX);
      tma_prefetch_desc(&mB);
      tma_prefetch_desc(&mC);
      int issued = 0;
      for (int c = 0; c < nch; ++c) {
        const int st = c & 1;
        if (c >= 2 && !wait1(s, &s.empty[st], ((c >> 1) + 1) & 1, p.status, 1)) break;
        mbar_expect_tx(&s.full[st], 5 * kQ * 128);
        const int tq = (cb + c) * kQ;
        tma_load_3d(s.C[st][0], &mC, &s.full[st], g * kN, tq, (int)b);
        tma_load_3d(s.C[st][1], &mC, &s.full[st], g * kN + 64, tq, (int)b);
        tma_load_3d(s.B[st][0], &mB, &s.full[st], g * kN, tq, (int)b);
        tma_load_3d(s.B[st][1], &mB, &s.full[st], g * kN + 64, tq, (int)b);
        tma_load_4d(s.X[st], &mX, &s.full[st], 0, (int)hd, tq, (int)b);
        issued = c + 1;
      }
      // Leave no copy in flight: the last two tiles issued have landed (a
      // phase already completed passes at once).
      for (int c = issued - 2; c < issued; ++c)
        if (c >= 0) mbar_wait(&s.full[c & 1], (c >> 1) & 1, kWaitLimit);
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (waits, descriptors: warp-uniform); one
    // elected lane issues the tcgen05 operations.
    const bool leader = elect_one();
    const uint32_t id_S = idesc_bf16_f32(128, 128, false, false);
    const uint32_t id_Y = idesc_bf16_f32(128, 64, false, true);
    const uint32_t id_Sc = idesc_bf16_f32(128, 64, true, true);
    // K-major C / B for S (16-byte K steps inside a slab, slabs 16 KB apart),
    // MN-major B / x / w o x / state copy (2 KB per 16-row K step).
    const uint64_t dCk[2] = {smem_desc(smem_u32(s.C[0][0]), 16, 1024, kSwizzle128B),
                             smem_desc(smem_u32(s.C[1][0]), 16, 1024, kSwizzle128B)};
    const uint64_t dBk[2] = {smem_desc(smem_u32(s.B[0][0]), 16, 1024, kSwizzle128B),
                             smem_desc(smem_u32(s.B[1][0]), 16, 1024, kSwizzle128B)};
    const uint64_t dBm[2] = {smem_desc(smem_u32(s.B[0][0]), kQ * 128, 1024, kSwizzle128B),
                             smem_desc(smem_u32(s.B[1][0]), kQ * 128, 1024, kSwizzle128B)};
    const uint64_t dX[2] = {smem_desc(smem_u32(s.X[0]), kQ * 128, 1024, kSwizzle128B),
                            smem_desc(smem_u32(s.X[1]), kQ * 128, 1024, kSwizzle128B)};
    const uint64_t dXw = smem_desc(smem_u32(s.Xw), kQ * 128, 1024, kSwizzle128B);
    const uint64_t dH[2] = {smem_desc(smem_u32(s.Hb[0]), kN * 128, 1024, kSwizzle128B),
                            smem_desc(smem_u32(s.Hb[1]), kN * 128, 1024, kSwizzle128B)};
    // (descriptor start addresses are in 16-byte units in the low 14 bits;
    // every operand lies below 232448 bytes, so adding an offset never
    // carries out of the field)
    uint64_t *last_bar = nullptr;  // barrier and phase parity of the last commit
    uint32_t last_par = 0;
    auto mma_S = [&](int c) {  // S(c) = C B^T into S[c & 1]
      const int st = c & 1;
      tc_fence_after();
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ko = ((kk >> 2) * (kQ * 128) + (kk & 3) * 32) >> 4;
          mma_ss(tb + kColS + 128 * st, dCk[st] + ko, dBk[st] + ko, id_S, kk > 0);
        }
        mma_commit(&s.sdone[st]);
      }
      __syncwarp();
      last_bar = &s.sdone[st];
      last_par = (c >> 1) & 1;
    };
    bool ok = nch > 0 && waitw(s, &s.full[0], 0, p.status, 2);
    if (ok) mma_S(0);
    for (int c = 0; ok && c < nch; ++c) {
      const int k = c & 1;
      const uint32_t ph = (c >> 1) & 1;
      // Sc(c) = B^T (w o x) once w o x of tile c is written, and S(c+1) once
      // the next tile has landed, in whichever order their inputs arrive
      // (both only have to follow Y(c-1)): the lanes poll both barriers
      // (bounded), and a barrier counts as passed when every lane has seen
      // it, so the warp decides together.
      bool need_sc = true, need_s = c + 1 < nch;
      const long long tw = clock64();
      while (need_sc || need_s) {
        if (need_sc && __all_sync(0xffffffffu, mbar_try(smem_u32(&s.xready[k]), ph))) {
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tb + kColSc + 64 * k, dBm[k] + kk * 128, dXw + kk * 128, id_Sc, kk > 0);
            mma_commit(&s.scdone[k]);
          }
          __syncwarp();
          last_bar = &s.scdone[k];
          last_par = ph;
          need_sc = false;
          continue;
        }
        if (need_s &&
            __all_sync(0xffffffffu, mbar_try(smem_u32(&s.full[k ^ 1]), ((c + 1) >> 1) & 1))) {
          mma_S(c + 1);
          need_s = false;
          continue;
        }
        if (__any_sync(0xffffffffu, clock64() - tw > kWaitLimit)) break;
      }
      if (need_sc || need_s) {
        if (lane == 0) set_abort(s, p.status, need_sc ? 3 : 4);
        break;
      }
      // Y(c) = M x + (e o C) h_prev: needs the mask group's operands, the
      // state of tile c-1 in Hb, and Y[k] read out by the output group
      if (!waitw(s, &s.mready[k], ph, p.status, 5)) break;
      if (c >= 1 && !waitw(s, &s.stdone[k ^ 1], ((c - 1) >> 1) & 1, p.status, 6)) break;
      if (c >= 2 && !waitw(s, &s.yfree[k], ((c - 2) >> 1) & 1, p.status, 7)) break;
      tc_fence_after();
      if (leader) {
        const uint32_t acol = tb + kColS + 128 * k, dcol = tb + kColY + 64 * k;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(dcol, acol + mask_col(kk >> 1, kk & 1), dX[k] + kk * 128, id_Y, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(dcol, acol + ec_col(kk), dH[k ^ 1] + kk * 128, id_Y, true);
        mma_commit(&s.yready[k]);
        mma_commit(&s.empty[k]);
      }
      __syncwarp();
      last_bar = &s.empty[k];
      last_par = ph;
    }
    // Leave no MMA in flight before TMEM is freed: wait (bounded) for the
    // barrier of the last commit issued, which tracks every earlier MMA.
    if (lane == 0 && last_bar) mbar_wait(last_bar, last_par, kWaitLimit);
    __syncwarp();
  } else if ((warp >= 4 && warp < 8) || (warp >= 14 && warp < 18)) {
    // ------------------------------------------------------------ mask group
    // Two warps per TMEM lane quarter (warps 4-7 and 14-17): each takes 32
    // rows and, of every row, half the work (16 of each 32-column block of
    // the mask, one 64-state slab of e o C).  Each warp keeps its own copy
    // of the tile's per-token factors, so the eight warps never wait for
    // each other; they meet only in the eight-count mready barrier.  They
    // do not read x: the output group forms w o x from the w_j published
    // here, so the convolution of the fused form runs beside S and the mask.
    const int half = warp >= 14 ? 1 : 0;
    const int mw = warp & 3;           // lane quarter = row block
    const int mg = 4 * half + mw;      // this warp's factor copy
    const int i = 32 * mw + lane;      // token of the tile; TMEM lane i
    const float A2 = p.A[hd] * kLog2e;
    const float bias = p.dt_bias ? p.dt_bias[hd] : 0.f;
    const float Dh = p.D ? p.D[hd] : 0.f;
    const bool softplus_on = p.flags & 1u;
    float *adw = s.adw[mg], *ppw = s.ppw[mg], *ddw = s.ddw[mg], *vdw = s.vdw[mg];
    // lane l handles tokens 4l .. 4l+3 of the tile in the prologue; their dt
    // is fetched a tile ahead and kept as raw bfloat16 bits until used
    const uint16_t *dtb = reinterpret_cast<const uint16_t *>(p.dt);
    uint32_t dtraw[4];
    auto fetch_dt = [&](int c) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t t = (int64_t)(cb + c) * kQ + 4 * lane + q;
        dtraw[q] = t < L ? (uint32_t)dtb[(b * L + t) * H + hd] : 0u;
      }
    };
    fetch_dt(0);
    for (int c = 0; c < nch; ++c) {
      const int k = c & 1;
      const int64_t t0 = (int64_t)(cb + c) * kQ;
      const int valid = (int)(L - t0 < kQ ? L - t0 : kQ);
      // The tile's step d_j and decay a_j = exp(d_j A) per token, and every
      // decay factor of the masked form as a product of the a_j -- never as
      // the exponential of a difference of running sums, whose rounding
      // would lose a token's small step beside a large sum (the "Mamba-2"
      // page's extreme A_h with a tiny step).  Within each 32-token block
      // (8 lanes): prefix products pp_j = a_b .. a_j and suffix products
      // a_{j+1} .. a_{b+31}; block totals T_K.  (Needs only dt, so it runs
      // while the tile's TMA is in flight.)
      float d4[4], a4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float d = 0.f;
        if (4 * lane + q < valid) {
          d = __uint_as_float(dtraw[q] << 16) + bias;
          if (softplus_on) d = softplus_sfu(d);
        }
        d4[q] = d;
        a4[q] = ex2(d * A2);
      }
      const float lp1 = a4[0] * a4[1], lp2 = lp1 * a4[2], lp3 = lp2 * a4[3];  // in-lane prefixes
      float incl = lp3;  // products over this lane and the earlier lanes of its block
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, incl, off, 8);
        if ((lane & 7) >= off) incl *= v;
      }
      float before = __shfl_up_sync(0xffffffffu, incl, 1, 8);
      if ((lane & 7) == 0) before = 1.f;
      float after = lp3;  // products over this lane and the later lanes of its block
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
        const float v = __shfl_down_sync(0xffffffffu, after, off, 8);
        if ((lane & 7) + off < 8) after *= v;
      }
      float later = __shfl_down_sync(0xffffffffu, after, 1, 8);
      if ((lane & 7) == 7) later = 1.f;
      const float T0 = __shfl_sync(0xffffffffu, incl, 7), T1 = __shfl_sync(0xffffffffu, incl, 15),
                  T2 = __shfl_sync(0xffffffffu, incl, 23), T3 = __shfl_sync(0xffffffffu, incl, 31);
      {
        const float pp[4] = {before * a4[0], before * lp1, before * lp2, before * lp3};
        const float sp[4] = {later * a4[3] * a4[2] * a4[1], later * a4[3] * a4[2], later * a4[3], later};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          adw[4 * lane + q] = a4[q];
          ppw[4 * lane + q] = pp[q];
          ddw[4 * lane + q] = d4[q];
          vdw[4 * lane + q] = sp[q] * d4[q];
        }
      }
      if (mg == 0 && lane == 0) s.a[c & 3] = T0 * T1 * T2 * T3;
      __syncwarp();
      // this row's factors: e_i = a_0 .. a_i and w_i = a_{i+1} .. a_127 d_i
      const float Tb[4] = {T0, T1, T2, T3};
      float before_blk = 1.f, after_blk = 1.f;
#pragma unroll
      for (int K = 0; K < 4; ++K) {
        if (K < mw) before_blk *= Tb[K];
        if (K > mw) after_blk *= Tb[K];
      }
      const float pp_i = ppw[i];
      const float e_i = pp_i * before_blk;
      const float w_i = vdw[i] * after_blk;
      // w_i for the output group's w o x (bf16, as the product uses it), and
      // with it the tile decay above: one arrival per half-0 warp
      if (half == 0) reinterpret_cast<uint16_t *>(s.wt[c & 3])[i] = (uint16_t)pack_bf16x2(w_i, 0.f);
      __syncwarp();
      if (half == 0 && lane == 0) mbar_arrive(&s.wready[c & 3]);
      // next tile's dt: it has the rest of this tile to arrive
      if (c + 1 < nch) fetch_dt(c + 1);
      // C of tile c (for e o C) has landed
      if (!waitw(s, &s.full[k], (c >> 1) & 1, p.status, 8)) break;
      // masked S -> bf16.  Of each 32-column block J this warp takes the 16
      // columns from 32 J + 16 half.  Its packed results go only where this
      // warp itself has already read S (its own halves of blocks 0 and 1),
      // so the pair never overwrites what the other still has to read:
      // block J -> packed columns mask_col(J, half) .. + 8, and the MMA
      // walks its K steps through the same map.
      if (!waitw(s, &s.sdone[k], (c >> 1) & 1, p.status, 10)) break;
      tc_fence_after();
      const uint32_t col = kColS + 128 * k;
#pragma unroll 1
      for (int J = 0; J < 4; ++J) {
        const int j0 = 32 * J + 16 * half;
        uint32_t r[16];
        uint32_t m[8];
        if (J <= mw) {
          tmem_ld16(tb + lane_base + col + j0, r);
          tmem_ld_wait();
        }
        if (J > mw) {
#pragma unroll
          for (int q = 0; q < 8; ++q) m[q] = 0u;
        } else if (J < mw) {
          // below the diagonal: S_ij * (a_{j+1} .. a_{32J+31}) d_j * u with
          // u = T_{J+1} .. T_{mw-1} (a_{32 mw} .. a_i); both factors <= 1 for
          // a decaying state
          float u = pp_i;
#pragma unroll
          for (int K = 1; K < 3; ++K)
            if (K > J && K < mw) u *= Tb[K];
          const float4 *vd4 = reinterpret_cast<const float4 *>(vdw + j0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 v = vd4[q];
            const f2 a = mul2(mul2(mk2(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])),
                                   mk2(v.x, v.y)),
                              mk2(u, u));
            const f2 bq = mul2(mul2(mk2(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])),
                                    mk2(v.z, v.w)),
                               mk2(u, u));
            m[2 * q] = pack_bf16x2(a.x, a.y);
            m[2 * q + 1] = pack_bf16x2(bq.x, bq.y);
          }
        } else {
          // diagonal block: S_ij * (a_{j+1} .. a_i) d_j for j <= i, + D at
          // j = i; the product runs down from j = i (exact, no cancellation)
          const int il = lane, jl0 = 16 * half;
          float P = 1.f;  // a_{jtop+1} .. a_i, jtop the last of this warp's columns <= i
          if (half == 0 && il >= 16) {
            const float4 *au = reinterpret_cast<const float4 *>(adw + 32 * J + 16);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const float4 a = au[v];
              if (16 + 4 * v <= il) P *= a.x;
              if (17 + 4 * v <= il) P *= a.y;
              if (18 + 4 * v <= il) P *= a.z;
              if (19 + 4 * v <= il) P *= a.w;
            }
          }
          const float4 *a4p = reinterpret_cast<const float4 *>(adw + j0);
          const float4 *d4p = reinterpret_cast<const float4 *>(ddw + j0);
#pragma unroll
          for (int q = 3; q >= 0; --q) {
            const float4 av = a4p[q], dv = d4p[q];
            const float as[4] = {av.x, av.y, av.z, av.w}, ds[4] = {dv.x, dv.y, dv.z, dv.w};
            float f[4];
#pragma unroll
            for (int e = 3; e >= 0; --e) {
              const int jl = jl0 + 4 * q + e;
              const float sv = __uint_as_float(r[4 * q + e]);
              if (jl <= il) {
                f[e] = sv * (P * ds[e]) + (jl == il ? Dh : 0.f);
                P *= as[e];
              } else {
                f[e] = 0.f;
              }
            }
            m[2 * q] = pack_bf16x2(f[0], f[1]);
            m[2 * q + 1] = pack_bf16x2(f[2], f[3]);
          }
        }
        tmem_st8(tb + lane_base + col + mask_col(J, half), m);
      }
      // e_i C_i -> bf16 for the states of slab `half`: 32 packed columns,
      // again only where this warp read S (its halves of blocks 2 and 3:
      // ec_col(2 c4 + kq) for K step kq of the slab); a warp that skipped
      // those blocks writes columns nobody reads S from.
      {
        const uint32_t e2 = pack_bf16x2(e_i, e_i);
#pragma unroll
        for (int c4 = 0; c4 < 2; ++c4) {
          uint32_t m[16];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 v = *reinterpret_cast<const uint4 *>(s.C[k][half] + sw128(i, 4 * c4 + q));
            m[4 * q] = bmul2(v.x, e2);
            m[4 * q + 1] = bmul2(v.y, e2);
            m[4 * q + 2] = bmul2(v.z, e2);
            m[4 * q + 3] = bmul2(v.w, e2);
          }
          tmem_st16(tb + lane_base + col + ec_col(4 * half + 2 * c4), m);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.mready[k]);
    }
  } else if (CONV && warp >= 18) {
    // ------------------------------------------------------------ convolution group
    // Fused form: the causal convolution of x over tokens, then silu, in
    // place in each landed tile, with nothing else to do, so it runs beside
    // the other roles.  Thread (cq, tg): channels 4 cq .. + 4 of the head,
    // tokens 32 tg .. + 32 of the tile, walked in order with the three
    // previous raw inputs in registers (every row read once); the three rows
    // before a tile are the previous tile's raw last rows (`halo`), or
    // before this CTA's first tile xBC's or the conv state's.  One barrier
    // between the reads a thread needs from its neighbour's rows and the
    // in-place writes; every wait is voted over the two warps.
    const int ci = tid - kThreads;
    const int cq = ci & 15, tg = ci >> 4;
    const uint32_t qoff = 8u * (uint32_t)(cq & 1);  // the quad within its 16-byte chunk
    const int64_t ch0 = hd * kP;
    auto waitc = [&](uint64_t *bar, uint32_t parity, int code) -> bool {
      const bool ok = mbar_wait(bar, parity, kWaitLimit);
      const bool fail = conv_group_any(!ok);
      if (fail && ci == 0) set_abort(s, p.status, code);
      return !fail;
    };
    // weights and bias of the thread's channels as pairs (0, 1), (2, 3)
    f2 wt3[2], wt2[2], wt1[2], wt0[2], bs[2];
    {
      const float4 *wv = reinterpret_cast<const float4 *>(p.cw + (ch0 + 4 * cq) * 4);
      const float4 w0 = __ldg(wv), w1 = __ldg(wv + 1), w2 = __ldg(wv + 2), w3 = __ldg(wv + 3);
      wt0[0] = mk2(w0.x, w1.x); wt1[0] = mk2(w0.y, w1.y); wt2[0] = mk2(w0.z, w1.z);
      wt3[0] = mk2(w0.w, w1.w);
      wt0[1] = mk2(w2.x, w3.x); wt1[1] = mk2(w2.y, w3.y); wt2[1] = mk2(w2.z, w3.z);
      wt3[1] = mk2(w2.w, w3.w);
      const float *bp = p.cbias + ch0 + 4 * cq;
      bs[0] = p.cbias ? mk2(__ldg(bp), __ldg(bp + 1)) : mk2(0.f, 0.f);
      bs[1] = p.cbias ? mk2(__ldg(bp + 2), __ldg(bp + 3)) : mk2(0.f, 0.f);
    }
    // Before this CTA's first tile the three preceding inputs come from
    // global memory, widened to float32 into the w o x buffer: the output
    // group writes it only after this group's first xconv arrival.
    const float *first = reinterpret_cast<const float *>(s.Xw);
    {
      const uint16_t *xr = reinterpret_cast<const uint16_t *>(p.xbc);
      const int64_t t0 = (int64_t)cb * kQ;
      for (int idx = ci; idx < 3 * kP; idx += kConvThreads) {
        const int row = idx / kP, ch = idx % kP;
        const int64_t tau = t0 - 3 + row;
        float v = 0.f;
        if (tau >= 0) v = __uint_as_float((uint32_t)xr[(b * L + tau) * p.ctot + ch0 + ch] << 16);
        else if (p.cs_in) v = p.cs_in[(b * p.ctot + ch0 + ch) * 3 + (tau + 3)];
        reinterpret_cast<float *>(s.Xw)[idx] = v;
      }
      conv_group_sync();
    }
    auto unpack2 = [](uint2 u, f2 (&v)[2]) {
      v[0] = mk2(bf16lo(u.x), bf16hi(u.x));
      v[1] = mk2(bf16lo(u.y), bf16hi(u.y));
    };
    const f2 half2 = mk2(0.5f, 0.5f);
    for (int c = 0; c < nch; ++c) {
      const int k = c & 1;
      const int64_t t0 = (int64_t)(cb + c) * kQ;
      if (!waitc(&s.full[k], (c >> 1) & 1, 16)) break;
      uint8_t *xs = s.X[k];
      f2 win[3][2];
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int r = 32 * tg - 3 + j;
        if (r >= 0) {
          unpack2(*reinterpret_cast<const uint2 *>(xs + sw128(r, cq >> 1) + qoff), win[j]);
        } else if (c > 0) {
          unpack2(*reinterpret_cast<const uint2 *>(&s.halo[r + 3][4 * cq]), win[j]);
        } else {
          const float4 f = *reinterpret_cast<const float4 *>(first + (r + 3) * kP + 4 * cq);
          win[j][0] = mk2(f.x, f.y);
          win[j][1] = mk2(f.z, f.w);
        }
      }
      conv_group_sync();  // every window is read: rows may be overwritten now
#pragma unroll 4
      for (int j = 0; j < 32; ++j) {
        const int r = 32 * tg + j;
        uint2 *row = reinterpret_cast<uint2 *>(xs + sw128(r, cq >> 1) + qoff);
        const uint2 u = *row;
        // the raw last three rows are the next tile's halo
        if (tg == 3 && j >= 29) *reinterpret_cast<uint2 *>(&s.halo[j - 29][4 * cq]) = u;
        f2 xv[2];
        unpack2(u, xv);
        // u = silu(bias + sum_q w[q] x[t - 3 + q]), the newest input first,
        // and silu(z) = z (1 + tanh(z / 2)) / 2: the operations of
        // ssm_conv1d_fwd lane by lane, so both give the same bits
        const bool live = t0 + r < L;
        uint32_t ov[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          f2 acc = fma2(wt3[q], xv[q], bs[q]);
          acc = fma2(wt2[q], win[2][q], acc);
          acc = fma2(wt1[q], win[1][q], acc);
          acc = fma2(wt0[q], win[0][q], acc);
          const f2 hz = mul2(half2, acc);
          float ta, tb2;
          asm("tanh.approx.f32 %0, %1;" : "=f"(ta) : "f"(hz.x));
          asm("tanh.approx.f32 %0, %1;" : "=f"(tb2) : "f"(hz.y));
          const f2 o = mul2(acc, fma2(half2, mk2(ta, tb2), half2));
          ov[q] = live ? pack_bf16x2(o.x, o.y) : 0u;
          win[0][q] = win[1][q];
          win[1][q] = win[2][q];
          win[2][q] = xv[q];
        }
        *row = make_uint2(ov[0], ov[1]);
      }
      // the convolved tile is read by the output group and, as Y's B
      // operand, by the tensor cores
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.xconv[k]);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ state group
    const int n = tid;
    float h[kP];
    {
      const float *src = h0u ? h0u + n * kP : nullptr;
#pragma unroll
      for (int q = 0; q < kP; q += 4) {
        const float4 v = src ? *reinterpret_cast<const float4 *>(src + q)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        h[q] = v.x; h[q + 1] = v.y; h[q + 2] = v.z; h[q + 3] = v.w;
      }
    }
    float dprod = 1.f;  // the segment's decay product (the carry's factor)
    for (int c = 0; c < nch; ++c) {
      const int k = c & 1;
      // h = a h + Sc (thread = row n); a comes from the mask group, whose
      // wready arrival orders its write before this read
      if (!waitw(s, &s.wready[c & 3], (c >> 2) & 1, p.status, 11)) break;
      if (!waitw(s, &s.scdone[k], (c >> 1) & 1, p.status, 12)) break;
      tc_fence_after();
      const float a_c = s.a[c & 3];
      dprod *= a_c;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        uint32_t r[16];
        tmem_ld16(tb + lane_base + kColSc + 64 * k + 16 * hh, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const f2 hn = fma2(mk2(a_c, a_c), mk2(h[16 * hh + j], h[16 * hh + j + 1]),
                             mk2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])));
          h[16 * hh + j] = hn.x;
          h[16 * hh + j + 1] = hn.y;
        }
      }
      tc_fence_before();
      // bf16 copy for Y(c+1); its previous contents (tile c-2) were read by
      // Y(c-1), which completed before Sc(c) (one issuer, in order)
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        *reinterpret_cast<uint4 *>(s.Hb[k] + sw128(n, cc)) =
            make_uint4(pack_bf16x2(h[8 * cc], h[8 * cc + 1]), pack_bf16x2(h[8 * cc + 2], h[8 * cc + 3]),
                       pack_bf16x2(h[8 * cc + 4], h[8 * cc + 5]),
                       pack_bf16x2(h[8 * cc + 6], h[8 * cc + 7]));
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.stdone[k]);
    }
    if (!aborted(s) && hlu) {
      float *dst = hlu + n * kP;
#pragma unroll
      for (int q = 0; q < kP; q += 4)
        *reinterpret_cast<float4 *>(dst + q) = make_float4(h[q], h[q + 1], h[q + 2], h[q + 3]);
    }
    if (!aborted(s) && decu && n == 0) *decu = dprod;
  } else {
    // ------------------------------------------------------------ output group
    const int i = tid - 256;  // token of the tile; TMEM lane i
    uint4 zr[8];
    auto load_z = [&](int c) {
      const int64_t t = (int64_t)(cb + c) * kQ + i;
      if (write_y && p.z && c < nch && t < L) {
        const __nv_bfloat16 *zp = p.z + ((b * L + t) * H + hd) * kP;
#pragma unroll
        for (int q = 0; q < 8; ++q) zr[q] = ld_cs_u4(zp + 8 * q);
      }
    };
    // w o x of tile c, the B operand of Sc(c) (thread = row), once x has
    // landed (fused: been convolved by the convolution group), the mask
    // group has published w_j and Sc(c-1) is done with the buffer.
    auto xprep = [&](int c) -> bool {
      const int k = c & 1;
      if (!waitw(s, CONV ? &s.xconv[k] : &s.full[k], (c >> 1) & 1, p.status, 14)) return false;
      if (!waitw(s, &s.wready[c & 3], (c >> 2) & 1, p.status, 15)) return false;
      if (c >= 1 && !waitw(s, &s.scdone[k ^ 1], ((c - 1) >> 1) & 1, p.status, 9)) return false;
      const uint32_t wb = reinterpret_cast<const uint16_t *>(s.wt[c & 3])[i];
      const uint32_t w2 = wb | (wb << 16);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const uint4 v = *reinterpret_cast<const uint4 *>(s.X[k] + sw128(i, cc));
        *reinterpret_cast<uint4 *>(s.Xw + sw128(i, cc)) =
            make_uint4(bmul2(v.x, w2), bmul2(v.y, w2), bmul2(v.z, w2), bmul2(v.w, w2));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.xready[k]);
      return true;
    };
    bool ok = nch > 0 && xprep(0);
    for (int c = 0; ok && c < nch; ++c) {
      const int k = c & 1;
      const int64_t t = (int64_t)(cb + c) * kQ + i;
      // the next tile's w o x first: Sc(c+1) waits for it while this tile's
      // Y is still being formed
      if (c + 1 < nch && !xprep(c + 1)) break;
      load_z(c);
      if (!waitw(s, &s.yready[k], (c >> 1) & 1, p.status, 13)) break;
      tc_fence_after();
      __nv_bfloat16 *yp = p.y + ((b * L + t) * H + hd) * kP;
      // two halves of 32 columns; Y[k] is released after the second load
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t v[32];
        tmem_ld16(tb + lane_base + kColY + 64 * k + 32 * hh, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
        tmem_ld16(tb + lane_base + kColY + 64 * k + 32 * hh + 16,
                  *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
        tmem_ld_wait();
        if (hh == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.yfree[k]);
        }
        if (write_y && t < L) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int q = 4 * hh + q4;
            float o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = __uint_as_float(v[8 * q4 + j]);
            if (p.z) {
              const uint32_t zw[4] = {zr[q].x, zr[q].y, zr[q].z, zr[q].w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                o[2 * j] *= silu_tanh(bf16lo(zw[j]));
                o[2 * j + 1] *= silu_tanh(bf16hi(zw[j]));
              }
            }
            st_cs_u4(yp + 8 * q, make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                            pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7])));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 13) tmem_dealloc(tb, kTmemCols);
}

// The state entering each segment of a tail unit: segment 0 started from the
// unit's own start state, so its end state is exact; the state is linear in
// the start state, so segment s's exact end is its end from zeros plus its
// decay product times the state that entered it.  Block = (tail unit, 1024
// of its N x P values); a thread carries four of them through the segments.
constexpr int kCarrySlice = 1024;
__global__ void __launch_bounds__(kCarrySlice / 4)
    ssd_seg_carry_kernel(const float *hend, const float *decay, float *hin, int nseg) {
  constexpr int kNP = kN * kP;
  pdl_launch_dependents();  // the whole units of the next launch may start
  const int64_t tu = blockIdx.x;
  const int e = blockIdx.y * kCarrySlice + threadIdx.x * 4;
  const float *he = hend + tu * nseg * kNP + e;
  const float *dc = decay + tu * nseg;
  float *hi = hin + tu * nseg * kNP + e;
  float4 h = *reinterpret_cast<const float4 *>(he);
#pragma unroll 4
  for (int sg = 1; sg < nseg; ++sg) {
    *reinterpret_cast<float4 *>(hi + (int64_t)sg * kNP) = h;
    if (sg + 1 < nseg) {
      const float4 l = *reinterpret_cast<const float4 *>(he + (int64_t)sg * kNP);
      const float d = dc[sg];
      h = make_float4(fmaf(d, h.x, l.x), fmaf(d, h.y, l.y), fmaf(d, h.z, l.z), fmaf(d, h.w, l.w));
    }
  }
}

constexpr int kBcRun = 8;  // tokens per thread in the B/C convolution pre-pass

// The fused call's pre-pass, one batch row per grid row (blockIdx.y).  (1)
// The B and C channels of xBC (nbc = 2 G N of them from channel c0 on)
// convolved over tokens, then silu, into bc [batch][L][nbc]: every head of a
// group reads the same B and C, so they are convolved once here instead of
// in each head's CTA (x is convolved inside the scan).  A thread takes
// eight channels over a run of tokens.  (2) The blocks after those: the conv state
// out, the last three inputs of every channel, oldest first (from cs_in
// where the sequence is shorter than three).  Indices within a row are
// 32-bit (the host keeps L * nbc / 8 and ctot below 2^31).
__global__ void __launch_bounds__(256)
    ssd_bc_conv_kernel(const __nv_bfloat16 *xbc, int64_t L, int64_t ctot, int64_t c0,
                       int nbc, unsigned conv_blocks, const float *cs_in, const float *cw,
                       const float *cbias, __nv_bfloat16 *bc, float *cs_out) {
  const int64_t bb = blockIdx.y;
  const unsigned nchunk = (unsigned)nbc / 8u;
  if (blockIdx.x < conv_blocks) {
    // thread = (8-channel chunk j, run of kBcRun tokens), walked in order
    // with the three previous inputs in registers
    const unsigned idx = blockIdx.x * 256u + threadIdx.x;
    const unsigned run = idx / nchunk, j = idx - run * nchunk;
    const int64_t t0 = (int64_t)run * kBcRun;
    if (t0 >= L) return;
    const int64_t ch = c0 + 8 * (int64_t)j;
    float w[8][4], bias[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(cw + (ch + e) * 4));
      w[e][0] = v.x; w[e][1] = v.y; w[e][2] = v.z; w[e][3] = v.w;
      bias[e] = cbias ? __ldg(cbias + ch + e) : 0.f;
    }
    float win[3][8];
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const int64_t tau = t0 - 3 + q;
      if (tau >= 0) {
        unpack8(ld_nc_u4(xbc + (bb * L + tau) * ctot + ch), win[q]);
      } else if (cs_in) {
#pragma unroll
        for (int e = 0; e < 8; ++e) win[q][e] = cs_in[(bb * ctot + ch + e) * 3 + (tau + 3)];
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) win[q][e] = 0.f;
      }
    }
    // every row of the run loaded before any is used (each thread's loads
    // in flight together, not one latency per token)
    uint4 raw[kBcRun];
#pragma unroll
    for (int r = 0; r < kBcRun; ++r)
      raw[r] = t0 + r < L ? ld_nc_u4(xbc + (bb * L + t0 + r) * ctot + ch) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int r = 0; r < kBcRun; ++r) {
      const int64_t t = t0 + r;
      if (t >= L) break;
      float xv[8];
      unpack8(raw[r], xv);
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {  // the newest input first, as ssm_conv1d_fwd
        float acc = fmaf(w[e][3], xv[e], bias[e]);
        acc = fmaf(w[e][2], win[2][e], acc);
        acc = fmaf(w[e][1], win[1][e], acc);
        acc = fmaf(w[e][0], win[0][e], acc);
        o[e] = silu_tanh(acc);
        win[0][e] = win[1][e];
        win[1][e] = win[2][e];
        win[2][e] = xv[e];
      }
      *reinterpret_cast<uint4 *>(bc + (bb * L + t) * nbc + 8 * j) =
          make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                     pack_bf16x2(o[6], o[7]));
    }
    return;
  }
  const unsigned c = (blockIdx.x - conv_blocks) * 256u + threadIdx.x;
  if (!cs_out || c >= (unsigned)ctot) return;
  const uint16_t *xr = reinterpret_cast<const uint16_t *>(xbc);
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    const int64_t tau = L - 3 + q;
    float v = 0.f;
    if (tau >= 0) v = __uint_as_float((uint32_t)xr[(bb * L + tau) * ctot + c] << 16);
    else if (cs_in) v = cs_in[(bb * ctot + c) * 3 + (tau + 3)];
    cs_out[(bb * ctot + c) * 3 + q] = v;
  }
}

bool encode(CUtensorMap *m, const void *ptr, int rank, const uint64_t *dims,
            const uint64_t *strides, const uint32_t *box) {
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, ptr, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool ssd_tc_supported(const M2Params &p) {
  return p.io == 1 && p.N == kN && p.P == kP && p.states == nullptr && p.H <= 65535 &&
         p.L < (1ll << 31) && p.batch <= 65535 && p.batch * p.H < (1ll << 31);
}

// One CTA per (batch, head) unit fills `sms` SMs a wave at a time; when the
// last wave is partial, its units are cut into segments that together fill
// one wave.  A cut pays for itself only with three segments or more (the
// segments run twice, once from zeros and once from the carried state), and
// a segment keeps at least four tiles.
SsdSplit ssd_tc_split(int64_t batch, int64_t H, int64_t L, int sms) {
  SsdSplit r;
  const int64_t units = batch * H, nch = (L + kQ - 1) / kQ;
  if (sms <= 0 || units <= 0) return r;
  const int64_t tail = units % sms;  // units of the partial wave (all, below one wave)
  if (tail == 0) return r;
  const int64_t nseg = std::min<int64_t>(sms / tail, nch / 4);
  if (nseg < 3) return r;
  r.ntail = tail;
  r.nseg = (int)nseg;
  return r;
}

size_t ssd_tc_split_bytes(const SsdSplit &r) {
  if (r.nseg <= 1) return 0;
  const size_t slots = (size_t)r.ntail * (size_t)r.nseg;
  return slots * (2 * (size_t)kN * kP + 4) * sizeof(float);
}

size_t ssd_tc_smem_bytes() { return sizeof(SsdSmem) + 1024; }

size_t ssd_conv_bc_bytes(int64_t batch, int64_t L, int64_t G) {
  return (size_t)(batch * L * 2 * G * kN) * sizeof(__nv_bfloat16);
}

cudaError_t launch_ssd_tc(const M2Params &p, int *status, const SsdSplit &split, void *seg_ws,
                          cudaStream_t stream, const SsdConv *conv) {
  const int64_t GN = p.G * kN;
  // x rows are H P channels apart, or, fused, xBC rows (ctot channels); B and
  // C rows G N apart, or, fused, the pre-pass's [B | C] rows (2 G N).
  const int64_t xrow = conv ? conv->ctot : p.H * kP;
  const int64_t bcrow = conv ? 2 * GN : GN;
  const void *xp = conv ? conv->xbc : p.x;
  const void *bp = conv ? conv->bc : p.B;
  const void *cp = conv ? static_cast<const void *>(static_cast<const __nv_bfloat16 *>(conv->bc) + GN)
                        : p.Cm;
  CUtensorMap mX, mB, mC;
  {
    uint64_t dims[4] = {(uint64_t)kP, (uint64_t)p.H, (uint64_t)p.L, (uint64_t)p.batch};
    uint64_t strides[3] = {(uint64_t)kP * 2, (uint64_t)(xrow * 2), (uint64_t)(p.L * xrow * 2)};
    uint32_t box[4] = {64, 1, kQ, 1};
    if (!encode(&mX, xp, 4, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[3] = {(uint64_t)GN, (uint64_t)p.L, (uint64_t)p.batch};
    uint64_t strides[2] = {(uint64_t)bcrow * 2, (uint64_t)(p.L * bcrow * 2)};
    uint32_t box[3] = {64, kQ, 1};
    if (!encode(&mB, bp, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!encode(&mC, cp, 3, dims, strides, box)) return cudaErrorInvalidValue;
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
  q.nfull = p.batch * p.H;
  q.tail0 = 0;
  q.ntail = 0;
  q.nseg = 1;
  q.seg_lo = 0;
  q.seg_hend = nullptr;
  q.seg_decay = nullptr;
  q.seg_hin = nullptr;
  q.xbc = conv ? static_cast<const __nv_bfloat16 *>(conv->xbc) : nullptr;
  q.ctot = conv ? conv->ctot : 0;
  q.cw = conv ? conv->w : nullptr;
  q.cbias = conv ? conv->bias : nullptr;
  q.cs_in = conv ? conv->state_in : nullptr;
  const size_t smem = ssd_tc_smem_bytes();
  auto kern = conv ? ssd_tc_kernel<true> : ssd_tc_kernel<false>;
  const int nthreads = conv ? threads_of<true>() : threads_of<false>();
  // (set on every call: the attribute belongs to the current device)
  {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (conv) {
    const unsigned conv_blocks =
        (unsigned)(((p.L + kBcRun - 1) / kBcRun * (2 * GN / 8) + 255) / 256);
    const unsigned state_blocks = conv->state_out ? (unsigned)((conv->ctot + 255) / 256) : 0u;
    ssd_bc_conv_kernel<<<dim3(conv_blocks + state_blocks, (unsigned)p.batch), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(conv->xbc), p.L, conv->ctot, p.H * kP, (int)(2 * GN),
        conv_blocks, conv->state_in, conv->w, conv->bias, static_cast<__nv_bfloat16 *>(conv->bc),
        conv->state_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (split.nseg <= 1) {
    kern<<<(unsigned)q.nfull, nthreads, smem, stream>>>(mX, mB, mC, q);
    return cudaGetLastError();
  }
  // Tail cut into segments: (1) every segment of the tail units from its own
  // start (the unit's start state for the first, zeros for the others),
  // (2) the carry, (3) the whole units and segments 1.. from the carried state.
  const int64_t units = q.nfull, slots = split.ntail * split.nseg;
  float *hend = static_cast<float *>(seg_ws);
  float *hin = hend + slots * kN * kP;
  float *dec = hin + slots * kN * kP;
  q.nfull = 0;
  q.tail0 = units - split.ntail;
  q.ntail = split.ntail;
  q.nseg = split.nseg;
  q.seg_hend = hend;
  q.seg_decay = dec;
  q.seg_hin = hin;
  kern<<<(unsigned)slots, nthreads, smem, stream>>>(mX, mB, mC, q);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ssd_seg_carry_kernel<<<dim3((unsigned)split.ntail, kN * kP / kCarrySlice), kCarrySlice / 4, 0,
                         stream>>>(hend, dec, hin, split.nseg);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  q.nfull = units - split.ntail;
  q.seg_lo = 1;
  // (a programmatic dependent of the carry: the whole units run while it does)
  return launch_dependent(kern, dim3((unsigned)(q.nfull + split.ntail * (split.nseg - 1))),
                          dim3(nthreads), smem, stream, mX, mB, mC, q);
}

}  // namespace ssm
