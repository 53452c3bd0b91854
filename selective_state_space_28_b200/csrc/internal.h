// internal.h -- launcher interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ssm.h"

namespace ssm {

// Mamba-1 scan, device pointers as in ssm_scan_args_t.
struct M1Params {
  int64_t batch, L, C, N, G;
  uint32_t flags;
  float eps;
  int io;  // 0 = f32, 1 = bf16
  const void *x, *dt, *z, *B, *Cm;
  const float *A, *D, *dt_bias, *h0;
  void *y;
  float *h_last, *states;
  float *rstd = nullptr;  // [batch * L] RMS factors of dt rows, or nullptr
  int *status = nullptr;  // device word set non-zero if a bounded wait ran out
  int64_t t_write = -1;                 // token whose state is replaced
  int part_base = 0;                    // a state write's first part in this launch
  const float *state_write = nullptr;   // [batch, C, N] state written at t_write
  // sequence segments of the pipelined kernel (nseg 1: the whole sequence)
  int nseg = 1;
  int64_t seg_len = 0;
  float *seg_end = nullptr;   // [nseg - 1, batch, C, N] end states from zero / h0
  float *seg_dsum = nullptr;  // [nseg - 1, batch, C] sums of the segments' steps
  float *seg_ent = nullptr;   // [nseg, batch, C, N] states entering each segment
};

// How the pipelined Mamba-1 kernel cuts the sequence (nseg 1: no cut).
struct M1Split {
  int nseg = 1;
  int64_t seg_len = 0;
};
M1Split m1_scan_split(int64_t batch, int64_t C, int64_t L, int64_t N, int sms);
size_t m1_scan_split_bytes(const M1Split &r, int64_t batch, int64_t C, int64_t N);
void m1_scan_split_carve(const M1Split &r, int64_t batch, int64_t C, int64_t N, void *ws,
                         M1Params &p);

// Mamba-2 token recurrence (the decode step, and the SSD path for shapes the
// chunked tensor-core kernel does not cover).
struct M2Params {
  int64_t batch, L, H, P, N, G;
  uint32_t flags;
  int io;
  const void *x, *z, *dt, *B, *Cm;
  const float *A, *D, *dt_bias;
  const float *h0;  // initial state or nullptr (the step passes its state)
  void *y;
  float *h_last, *states;
};

struct M1StepParams {
  int64_t batch, C, N, G;
  uint32_t flags;
  float eps;
  int io;
  const void *x, *dt, *z, *B, *Cm;
  const float *A, *D, *dt_bias;
  float *state;
  void *y;
};

// Causal depthwise convolution over tokens (then silu when `silu`).
constexpr int kConvMaxWidth = 4;
struct ConvParams {
  int64_t batch, L, Cc;
  int W;
  int io;
  bool silu;
  int64_t run;  // tokens per thread (conv1d_run_length)
  const void *x;
  const float *w, *bias, *state_in;
  void *u;
  float *state_out;
};

// The Mamba-2 mixer's gated RMS norm over rows of `width` values.
constexpr int64_t kGatedNormMaxWidth = 49152;  // the row lives in shared memory
struct GatedNormParams {
  int64_t rows, width;
  int io;
  float eps;
  const void *y, *z;
  const float *weight;
  void *out;
};

// The hidden attention of the SSD map, exported as [b, H, L, L] float32.
struct AttnParams {
  int64_t batch, L, H, N, G;
  uint32_t flags;
  int io;
  int heads_per_cta;
  const void *dt, *B, *Cm;
  const float *A, *dt_bias;
  float *alpha;
  float *beta;   // workspace: [b, H, L] steps
  double *cum;   // workspace: [b, H, L] running log2-decay sums
  float *cb;     // workspace: [b, G, ntri, 128, 128] C . B^T of the lower tiles
  int64_t ntri;  // tiles on or below the diagonal
};

// Each returns cudaSuccess, cudaErrorNotSupported for a shape without a
// kernel (checked before any launch), or the launch error.
cudaError_t launch_m1_scan(const M1Params &p, cudaStream_t s);
bool m1_scan_supported(int64_t N, int64_t C, int64_t G);
bool m1_scan_tma_supported(const M1Params &p);
cudaError_t launch_m1_scan_tma(const M1Params &p, cudaStream_t s);
cudaError_t launch_m2_recurrent(const M2Params &p, cudaStream_t s);
bool m2_recurrent_supported(int64_t N, int64_t P);
cudaError_t launch_m1_step(const M1StepParams &p, cudaStream_t s);
bool m1_step_supported(int64_t N);
// Tensor-core SSD (bf16 I/O, state 128, head dim 64, no per-token states).
// `status` is a device word the kernel sets non-zero if a bounded wait ran out.
bool ssd_tc_supported(const M2Params &p);
// How the tensor-core SSD cuts the (batch, head) units of a partial last wave
// into sequence segments (nseg == 1: no cut), and the workspace that takes.
struct SsdSplit {
  int64_t ntail = 0;
  int nseg = 1;
};
SsdSplit ssd_tc_split(int64_t batch, int64_t H, int64_t L, int sms);
size_t ssd_tc_split_bytes(const SsdSplit &r);
int device_sm_count();  // the current device's SMs (148 when it cannot be read)
int64_t conv1d_run_length(const ConvParams &p, bool state_in_place);
bool conv1d_supported(const ConvParams &p);
bool gated_norm_supported(const GatedNormParams &p);
int attn_heads_per_cta(int64_t H, int64_t G);
bool attention_supported(const AttnParams &p);
size_t attention_workspace_bytes(int64_t batch, int64_t H, int64_t G, int64_t L);
int64_t attention_lower_tiles(int64_t L);
cudaError_t launch_attention(const AttnParams &p, cudaStream_t s);
cudaError_t launch_gated_norm(const GatedNormParams &p, cudaStream_t s);
cudaError_t launch_conv1d(const ConvParams &p, cudaStream_t s);
// The Mamba-2 mixer's causal convolution fused into the tensor-core SSD:
// x, B and C come from xBC [batch][L][ctot] (bf16, before the convolution,
// ctot = H P + 2 G N), convolved with w [ctot][4] and bias, then silu; the
// three inputs before token 0 from state_in [batch][ctot][3] or zeros;
// state_out receives the last three inputs.  bc is workspace for the
// convolved B and C (ssd_conv_bc_bytes).
struct SsdConv {
  const void *xbc;
  int64_t ctot;
  const float *w, *bias, *state_in;
  float *state_out;
  void *bc;
};
size_t ssd_conv_bc_bytes(int64_t batch, int64_t L, int64_t G);
cudaError_t launch_ssd_tc(const M2Params &p, int *status, const SsdSplit &split, void *seg_ws,
                          cudaStream_t s, const SsdConv *conv = nullptr);

// The Mamba-1 scan behind ssm_scan_fwd, ssm_scan_fwd_write (t_write >= 0)
// and ssm_scan_fwd_static (allow_cut false: the sequence is never cut into
// segments, so the workspace is the status word and the dt-norm factors).
// reset_status false leaves the status word as it is (a caller that runs
// several scans against one status word clears it once).
ssm_status_t scan_run(const ssm_scan_args_t *a, int64_t t_write, const float *state_write,
                      void *stream, bool allow_cut, bool reset_status = true);
// The workspace bytes scan_run needs for these shapes and flags (pointers
// not looked at; allow_cut as in scan_run).
size_t scan_workspace_bytes(const ssm_scan_args_t *a, bool allow_cut);
// Every host-side check of ssm_scan_fwd (pointers included), touching no
// device: SSM_OK or the error status.
ssm_status_t scan_validate(const ssm_scan_args_t *a);
// Device address of the allocation-free entry point's static scratch on the
// current device (its first word is that entry point's status word).
cudaError_t static_scratch_address(void **out);

}  // namespace ssm
