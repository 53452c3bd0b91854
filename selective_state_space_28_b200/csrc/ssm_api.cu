// ssm_api.cu -- the exported C ABI (include/ssm.h): argument validation on
// the host, then dispatch to the kernels.  Nothing is launched when a check
// fails, and nothing here allocates memory.
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "internal.h"
#include "ssm.h"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Every non-NULL pointer must be 16-byte aligned.
template <typename... Ps>
bool all_aligned(Ps... ps) {
  const void *arr[] = {static_cast<const void *>(ps)...};
  for (const void *p : arr)
    if (p && !aligned16(p)) return false;
  return true;
}

}  // namespace

namespace ssm {
int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();  // (no device here: size for a B200)
    return 148;
  }
  return n;
}
}  // namespace ssm

namespace {

ssm_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return SSM_OK;
  if (e == cudaErrorNotSupported) return SSM_ERR_UNSUPPORTED;
  return SSM_ERR_CUDA;
}

// seqlen == 0: the state passes through unchanged (h_last = h0, or zeros).
ssm_status_t pass_state(const float *h0, float *h_last, size_t bytes, cudaStream_t s) {
  if (!h_last || bytes == 0) return SSM_OK;
  cudaError_t e = cudaSuccess;
  if (!h0) e = cudaMemsetAsync(h_last, 0, bytes, s);
  else if (h0 != h_last) e = cudaMemcpyAsync(h_last, h0, bytes, cudaMemcpyDeviceToDevice, s);
  return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// The Mamba-1 workspace: a status word (256 bytes), the dt-norm factors
// (batch * seqlen floats, with SSM_RMSNORM_DT), then the sequence segments'
// states when the call is cut.  `cut` false keeps the whole sequence in one
// pass (the allocation-free entry point).
constexpr size_t kStatusBytes = 256;
struct M1Layout {
  size_t rstd_off = 0, seg_off = 0, total = 0;
  ssm::M1Split split;
};
size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }
bool m1_cut_allowed(const ssm_scan_args_t *a) { return !a->states; }
M1Layout m1_layout(const ssm_scan_args_t *a, int sms, bool cut = true) {
  M1Layout l;
  l.rstd_off = kStatusBytes;
  const size_t rstd = (a->flags & SSM_RMSNORM_DT) ? (size_t)(a->batch * a->seqlen) * sizeof(float) : 0;
  l.seg_off = l.rstd_off + round256(rstd);
  ssm::M1Params probe;
  probe.batch = a->batch;
  probe.L = a->seqlen;
  probe.C = a->channels;
  probe.N = a->state;
  probe.G = a->groups;
  probe.io = a->io;
  if (cut && m1_cut_allowed(a) && a->batch > 0 && a->seqlen > 0 &&
      ssm::m1_scan_tma_supported(probe))
    l.split = ssm::m1_scan_split(a->batch, a->channels, a->seqlen, a->state, sms);
  l.total = l.seg_off + ssm::m1_scan_split_bytes(l.split, a->batch, a->channels, a->state);
  return l;
}

// shapes_only: the workspace query validates sizes and flags, not pointers.
ssm_status_t check_scan(const ssm_scan_args_t *a, size_t *ws, bool shapes_only = false,
                        bool size_it = true) {
  if (!a) return SSM_ERR_NULL;
  if (a->io != SSM_F32 && a->io != SSM_BF16) return SSM_ERR_DTYPE;
  if (a->batch < 0 || a->seqlen < 0 || a->channels <= 0 || a->state <= 0 ||
      a->groups <= 0 || a->channels % a->groups)
    return SSM_ERR_SHAPE;
  if (a->flags & ~(SSM_DT_SOFTPLUS | SSM_RMSNORM_BC | SSM_RMSNORM_DT))
    return SSM_ERR_UNSUPPORTED;
  if ((a->flags & (SSM_RMSNORM_BC | SSM_RMSNORM_DT)) && !(a->rms_eps >= 0.f))
    return SSM_ERR_SHAPE;
  if (!shapes_only && a->batch > 0 && a->seqlen > 0 &&
      (!a->x || !a->dt || !a->B || !a->C || !a->A || !a->y))
    return SSM_ERR_NULL;
  if (!shapes_only &&
      !all_aligned(a->x, a->dt, a->z, a->B, a->C, a->A, a->D, a->dt_bias, a->h0, a->y,
                   a->h_last, a->states, a->workspace))
    return SSM_ERR_ALIGN;
  if (!ssm::m1_scan_supported(a->state, a->channels, a->groups) || a->batch > 65535)
    return SSM_ERR_UNSUPPORTED;
  if (size_it) *ws = m1_layout(a, ssm::device_sm_count()).total;
  return SSM_OK;
}

// The tensor-core SSD path keeps a device status word at the start of the
// workspace, then (when the last wave's units are cut into segments) the
// segments' end states, carried states and decay products.
constexpr size_t kSsdStatusBytes = 256;

ssm::M2Params ssd_params(const ssd_scan_args_t *a) {
  ssm::M2Params p;
  p.batch = a->batch;
  p.L = a->seqlen;
  p.H = a->heads;
  p.P = a->head_dim;
  p.N = a->state;
  p.G = a->groups;
  p.flags = a->flags;
  p.io = a->io;
  p.x = a->x;
  p.z = a->z;
  p.dt = a->dt;
  p.B = a->B;
  p.Cm = a->C;
  p.A = a->A;
  p.D = a->D;
  p.dt_bias = a->dt_bias;
  p.h0 = a->h0;
  p.y = a->y;
  p.h_last = a->h_last;
  p.states = a->states;
  return p;
}

ssm_status_t check_ssd(const ssd_scan_args_t *a, size_t *ws, bool shapes_only = false) {
  if (!a) return SSM_ERR_NULL;
  if (a->io != SSM_F32 && a->io != SSM_BF16) return SSM_ERR_DTYPE;
  if (a->batch < 0 || a->seqlen < 0 || a->heads <= 0 || a->head_dim <= 0 ||
      a->state <= 0 || a->groups <= 0 || a->chunk <= 0 || a->heads % a->groups)
    return SSM_ERR_SHAPE;
  if (a->flags & ~SSM_DT_SOFTPLUS) return SSM_ERR_UNSUPPORTED;
  if (!shapes_only && a->batch > 0 && a->seqlen > 0 &&
      (!a->x || !a->dt || !a->B || !a->C || !a->A || !a->y))
    return SSM_ERR_NULL;
  if (!shapes_only &&
      !all_aligned(a->x, a->z, a->dt, a->B, a->C, a->A, a->D, a->dt_bias, a->h0, a->y,
                   a->h_last, a->states, a->workspace))
    return SSM_ERR_ALIGN;
  if (!ssm::m2_recurrent_supported(a->state, a->head_dim) || a->batch > 65535)
    return SSM_ERR_UNSUPPORTED;
  *ws = ssm::ssd_tc_supported(ssd_params(a))
            ? kSsdStatusBytes + ssm::ssd_tc_split_bytes(ssm::ssd_tc_split(
                                    a->batch, a->heads, a->seqlen, ssm::device_sm_count()))
            : 0;
  return SSM_OK;
}

// The fused convolution + SSD: the tensor-core configuration only.  The
// workspace holds the status word, the convolved B and C, then the segment
// states of a cut last wave.
struct SsdConvLayout {
  size_t bc_off = 0, seg_off = 0, total = 0;
};

SsdConvLayout ssd_conv_layout(const ssd_conv_scan_args_t *a, int sms) {
  const auto r256 = [](size_t v) { return (v + 255) & ~(size_t)255; };
  SsdConvLayout l;
  l.bc_off = kSsdStatusBytes;
  l.seg_off = l.bc_off + r256(ssm::ssd_conv_bc_bytes(a->batch, a->seqlen, a->groups));
  l.total = l.seg_off + ssm::ssd_tc_split_bytes(ssm::ssd_tc_split(a->batch, a->heads, a->seqlen, sms));
  return l;
}

ssm_status_t check_ssd_conv(const ssd_conv_scan_args_t *a, size_t *ws, bool shapes_only) {
  if (!a) return SSM_ERR_NULL;
  if (a->io != SSM_F32 && a->io != SSM_BF16) return SSM_ERR_DTYPE;
  if (a->batch < 0 || a->seqlen < 0 || a->heads <= 0 || a->head_dim <= 0 ||
      a->state <= 0 || a->groups <= 0 || a->chunk <= 0 || a->heads % a->groups)
    return SSM_ERR_SHAPE;
  if (a->flags & ~SSM_DT_SOFTPLUS) return SSM_ERR_UNSUPPORTED;
  // (the convolution pre-pass indexes a batch row's tokens x 8-channel
  // chunks in 32 bits)
  if (a->io != SSM_BF16 || a->state != 128 || a->head_dim != 64 || a->batch > 65535 ||
      a->heads > 65535 || a->batch * a->heads >= (1ll << 31) ||
      a->seqlen * a->groups * 32 >= (1ll << 31))
    return SSM_ERR_UNSUPPORTED;
  const int64_t ctot = a->heads * a->head_dim + 2 * a->groups * a->state;
  if (!shapes_only && a->batch > 0 && a->seqlen > 0 &&
      (!a->xBC || !a->conv_w || !a->dt || !a->A || !a->y))
    return SSM_ERR_NULL;
  if (!shapes_only &&
      !all_aligned(a->xBC, a->conv_w, a->conv_bias, a->conv_state_in, a->conv_state_out, a->z,
                   a->dt, a->A, a->D, a->dt_bias, a->h0, a->y, a->h_last, a->workspace))
    return SSM_ERR_ALIGN;
  if (!shapes_only && a->conv_state_in && a->conv_state_out) {
    const uintptr_t i0 = reinterpret_cast<uintptr_t>(a->conv_state_in);
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(a->conv_state_out);
    const uintptr_t n = (uintptr_t)(a->batch * ctot * 3) * sizeof(float);
    if (n && i0 < o0 + n && o0 < i0 + n) return SSM_ERR_SHAPE;
  }
  *ws = ssd_conv_layout(a, ssm::device_sm_count()).total;
  return SSM_OK;
}

}  // namespace

namespace ssm {

ssm_status_t scan_validate(const ssm_scan_args_t *a) {
  size_t ws = 0;
  return check_scan(a, &ws, false, false);
}

size_t scan_workspace_bytes(const ssm_scan_args_t *a, bool allow_cut) {
  return m1_layout(a, device_sm_count(), allow_cut).total;
}

ssm_status_t scan_run(const ssm_scan_args_t *a, int64_t t_write, const float *state_write,
                      void *stream, bool allow_cut, bool reset_status) {
  size_t ws = 0;
  ssm_status_t st = check_scan(a, &ws);
  if (st != SSM_OK) return st;
  if (a->batch == 0) return SSM_OK;  // nothing to do, nothing launched
  const M1Layout lay = m1_layout(a, device_sm_count(), allow_cut && t_write < 0);
  if (!a->workspace || a->workspace_bytes < lay.total) return SSM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int *status = static_cast<int *>(a->workspace);
  if (reset_status && cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess)
    return SSM_ERR_CUDA;
  if (a->seqlen == 0)
    return pass_state(a->h0, a->h_last,
                      (size_t)(a->batch * a->channels * a->state) * sizeof(float), s);
  M1Params p;
  p.batch = a->batch;
  p.L = a->seqlen;
  p.C = a->channels;
  p.N = a->state;
  p.G = a->groups;
  p.flags = a->flags;
  p.eps = a->rms_eps;
  p.io = a->io;
  p.x = a->x;
  p.dt = a->dt;
  p.z = a->z;
  p.B = a->B;
  p.Cm = a->C;
  p.A = a->A;
  p.D = a->D;
  p.dt_bias = a->dt_bias;
  p.h0 = a->h0;
  p.y = a->y;
  p.h_last = a->h_last;
  p.states = a->states;
  char *w = static_cast<char *>(a->workspace);
  p.rstd = (a->flags & SSM_RMSNORM_DT) ? reinterpret_cast<float *>(w + lay.rstd_off) : nullptr;
  p.status = status;
  p.t_write = t_write;
  p.state_write = state_write;
  m1_scan_split_carve(lay.split, a->batch, a->channels, a->state, w + lay.seg_off, p);
  if (p.nseg <= 1) p.seg_len = a->seqlen;
  return from_cuda(launch_m1_scan(p, s));
}

}  // namespace ssm

extern "C" {

int ssm_abi_version(void) { return SSM_ABI_VERSION; }

const char *ssm_status_string(ssm_status_t s) {
  switch (s) {
    case SSM_OK: return "ok";
    case SSM_ERR_NULL: return "a required pointer is NULL";
    case SSM_ERR_SHAPE: return "invalid size or shape";
    case SSM_ERR_DTYPE: return "unsupported io dtype";
    case SSM_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SSM_ERR_UNSUPPORTED: return "combination the library has no kernel for";
    case SSM_ERR_WORKSPACE: return "workspace missing or too small";
    case SSM_ERR_CUDA: return "CUDA error";
    case SSM_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

ssm_status_t ssm_scan_workspace(const ssm_scan_args_t *a, size_t *bytes) {
  if (!bytes) return SSM_ERR_NULL;
  size_t ws = 0;
  ssm_status_t st = check_scan(a, &ws, true);
  if (st == SSM_OK) *bytes = ws;
  return st;
}

ssm_status_t ssm_scan_fwd(const ssm_scan_args_t *a, void *stream) {
  return ssm::scan_run(a, -1, nullptr, stream, true);
}

ssm_status_t ssm_scan_fwd_write(const ssm_scan_args_t *a, int64_t t_write,
                                const float *state_write, void *stream) {
  if (a && a->batch > 0 && !state_write) return SSM_ERR_NULL;
  if (!all_aligned(state_write)) return SSM_ERR_ALIGN;
  if (a && (t_write < 0 || t_write >= a->seqlen)) return SSM_ERR_SHAPE;
  return ssm::scan_run(a, t_write, state_write, stream, true);
}

ssm_status_t ssm_workspace_status(const void *workspace, void *stream) {
  if (!workspace) {
    void *scratch = nullptr;
    if (ssm::static_scratch_address(&scratch) != cudaSuccess) return SSM_ERR_CUDA;
    workspace = scratch;
  }
  int word = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SSM_ERR_CUDA;
  return word ? SSM_ERR_TIMEOUT : SSM_OK;
}

ssm_status_t ssd_chunk_scan_workspace(const ssd_scan_args_t *a, size_t *bytes) {
  if (!bytes) return SSM_ERR_NULL;
  size_t ws = 0;
  ssm_status_t st = check_ssd(a, &ws, true);
  if (st == SSM_OK) *bytes = ws;
  return st;
}

ssm_status_t ssd_chunk_scan_fwd(const ssd_scan_args_t *a, void *stream) {
  size_t ws = 0;
  ssm_status_t st = check_ssd(a, &ws);
  if (st != SSM_OK) return st;
  if (a->batch == 0) return SSM_OK;  // nothing to do, nothing launched
  if (ws && (!a->workspace || a->workspace_bytes < ws)) return SSM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->seqlen == 0)
    return pass_state(a->h0, a->h_last,
                      (size_t)(a->batch * a->heads * a->state * a->head_dim) * sizeof(float),
                      s);
  const ssm::M2Params p = ssd_params(a);
  if (ssm::ssd_tc_supported(p)) {
    int *status = static_cast<int *>(a->workspace);
    if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return SSM_ERR_CUDA;
    const ssm::SsdSplit split =
        ssm::ssd_tc_split(a->batch, a->heads, a->seqlen, ssm::device_sm_count());
    return from_cuda(ssm::launch_ssd_tc(p, status, split,
                                        static_cast<char *>(a->workspace) + kSsdStatusBytes, s));
  }
  return from_cuda(ssm::launch_m2_recurrent(p, s));
}

ssm_status_t ssd_conv_chunk_scan_workspace(const ssd_conv_scan_args_t *a, size_t *bytes) {
  if (!bytes) return SSM_ERR_NULL;
  size_t ws = 0;
  ssm_status_t st = check_ssd_conv(a, &ws, true);
  if (st == SSM_OK) *bytes = ws;
  return st;
}

ssm_status_t ssd_conv_chunk_scan_fwd(const ssd_conv_scan_args_t *a, void *stream) {
  size_t ws = 0;
  ssm_status_t st = check_ssd_conv(a, &ws, false);
  if (st != SSM_OK) return st;
  if (a->batch == 0) return SSM_OK;  // nothing to do, nothing launched
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t ctot = a->heads * a->head_dim + 2 * a->groups * a->state;
  if (a->seqlen == 0) {  // both states pass through unchanged
    st = pass_state(a->h0, a->h_last,
                    (size_t)(a->batch * a->heads * a->state * a->head_dim) * sizeof(float), s);
    if (st != SSM_OK) return st;
    return pass_state(a->conv_state_in, a->conv_state_out,
                      (size_t)(a->batch * ctot * 3) * sizeof(float), s);
  }
  if (!a->workspace || a->workspace_bytes < ws) return SSM_ERR_WORKSPACE;
  const int sms = ssm::device_sm_count();
  const SsdConvLayout l = ssd_conv_layout(a, sms);
  ssm::M2Params p;
  p.batch = a->batch;
  p.L = a->seqlen;
  p.H = a->heads;
  p.P = a->head_dim;
  p.N = a->state;
  p.G = a->groups;
  p.flags = a->flags;
  p.io = a->io;
  p.x = nullptr;
  p.z = a->z;
  p.dt = a->dt;
  p.B = nullptr;
  p.Cm = nullptr;
  p.A = a->A;
  p.D = a->D;
  p.dt_bias = a->dt_bias;
  p.h0 = a->h0;
  p.y = a->y;
  p.h_last = a->h_last;
  p.states = nullptr;
  ssm::SsdConv conv;
  conv.xbc = a->xBC;
  conv.ctot = ctot;
  conv.w = a->conv_w;
  conv.bias = a->conv_bias;
  conv.state_in = a->conv_state_in;
  conv.state_out = a->conv_state_out;
  char *w = static_cast<char *>(a->workspace);
  conv.bc = w + l.bc_off;
  int *status = reinterpret_cast<int *>(w);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return SSM_ERR_CUDA;
  const ssm::SsdSplit split = ssm::ssd_tc_split(a->batch, a->heads, a->seqlen, sms);
  return from_cuda(ssm::launch_ssd_tc(p, status, split, w + l.seg_off, s, &conv));
}

ssm_status_t ssm_scan_step(const ssm_step_args_t *a, void *stream) {
  if (!a) return SSM_ERR_NULL;
  if (a->io != SSM_F32 && a->io != SSM_BF16) return SSM_ERR_DTYPE;
  if (a->kind != SSM_STEP_MAMBA1 && a->kind != SSM_STEP_MAMBA2) return SSM_ERR_UNSUPPORTED;
  if (a->batch < 0 || a->units <= 0 || a->head_dim <= 0 || a->state <= 0 ||
      a->groups <= 0 || a->units % a->groups)
    return SSM_ERR_SHAPE;
  if (a->kind == SSM_STEP_MAMBA1 && a->head_dim != 1) return SSM_ERR_SHAPE;
  const uint32_t allowed =
      a->kind == SSM_STEP_MAMBA1 ? (SSM_DT_SOFTPLUS | SSM_RMSNORM_BC) : SSM_DT_SOFTPLUS;
  if (a->flags & ~allowed) return SSM_ERR_UNSUPPORTED;
  if ((a->flags & SSM_RMSNORM_BC) && !(a->rms_eps >= 0.f)) return SSM_ERR_SHAPE;
  if (a->batch > 0 && (!a->x || !a->dt || !a->B || !a->C || !a->A || !a->state_io || !a->y))
    return SSM_ERR_NULL;
  if (!all_aligned(a->x, a->dt, a->z, a->B, a->C, a->A, a->D, a->dt_bias, a->state_io, a->y))
    return SSM_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->kind == SSM_STEP_MAMBA1) {
    if (!ssm::m1_step_supported(a->state)) return SSM_ERR_UNSUPPORTED;
    if (a->batch == 0) return SSM_OK;
    ssm::M1StepParams p;
    p.batch = a->batch;
    p.C = a->units;
    p.N = a->state;
    p.G = a->groups;
    p.flags = a->flags;
    p.eps = a->rms_eps;
    p.io = a->io;
    p.x = a->x;
    p.dt = a->dt;
    p.z = a->z;
    p.B = a->B;
    p.Cm = a->C;
    p.A = a->A;
    p.D = a->D;
    p.dt_bias = a->dt_bias;
    p.state = a->state_io;
    p.y = a->y;
    return from_cuda(ssm::launch_m1_step(p, s));
  }
  if (!ssm::m2_recurrent_supported(a->state, a->head_dim) || a->batch > 65535)
    return SSM_ERR_UNSUPPORTED;
  if (a->batch == 0) return SSM_OK;
  ssm::M2Params p;
  p.batch = a->batch;
  p.L = 1;
  p.H = a->units;
  p.P = a->head_dim;
  p.N = a->state;
  p.G = a->groups;
  p.flags = a->flags;
  p.io = a->io;
  p.x = a->x;
  p.z = a->z;
  p.dt = a->dt;
  p.B = a->B;
  p.Cm = a->C;
  p.A = a->A;
  p.D = a->D;
  p.dt_bias = a->dt_bias;
  p.h0 = a->state_io;
  p.y = a->y;
  p.h_last = a->state_io;
  p.states = nullptr;
  return from_cuda(ssm::launch_m2_recurrent(p, s));
}

ssm_status_t ssm_conv1d_fwd(const ssm_conv_args_t *a, void *stream) {
  if (!a) return SSM_ERR_NULL;
  if (a->io != SSM_F32 && a->io != SSM_BF16) return SSM_ERR_DTYPE;
  if (a->batch < 0 || a->seqlen < 0 || a->channels <= 0 || a->width <= 0) return SSM_ERR_SHAPE;
  if (a->width > ssm::kConvMaxWidth || (a->flags & ~SSM_CONV_SILU)) return SSM_ERR_UNSUPPORTED;
  if (!a->w) return SSM_ERR_NULL;
  const bool work = a->batch > 0 && a->seqlen > 0;
  if (work && (!a->x || !a->u)) return SSM_ERR_NULL;
  if (!all_aligned(a->x, a->u, a->w, a->bias, a->state_in, a->state_out)) return SSM_ERR_ALIGN;
  const size_t esz = a->io == SSM_BF16 ? 2 : 4;
  const size_t xbytes = (size_t)a->batch * a->seqlen * a->channels * esz;
  const size_t sbytes = (size_t)a->batch * a->channels * (a->width - 1) * sizeof(float);
  // x and u must not overlap; the state may be updated in place, nothing else
  auto overlap = [](const void *p, const void *q, size_t n) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p), b0 = reinterpret_cast<uintptr_t>(q);
    return n > 0 && a0 < b0 + n && b0 < a0 + n;
  };
  if (work && overlap(a->x, a->u, xbytes)) return SSM_ERR_SHAPE;
  const bool in_place = a->state_in && a->state_out == a->state_in;
  if (a->state_in && a->state_out && !in_place && overlap(a->state_in, a->state_out, sbytes))
    return SSM_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->batch == 0) return SSM_OK;
  if (a->seqlen == 0) return pass_state(a->state_in, a->state_out, sbytes, s);
  ssm::ConvParams p;
  p.batch = a->batch;
  p.L = a->seqlen;
  p.Cc = a->channels;
  p.W = (int)a->width;
  p.io = a->io;
  p.silu = (a->flags & SSM_CONV_SILU) != 0;
  p.x = a->x;
  p.w = a->w;
  p.bias = a->bias;
  p.state_in = a->state_in;
  p.u = a->u;
  p.state_out = a->width > 1 ? a->state_out : nullptr;
  p.run = ssm::conv1d_run_length(p, in_place);
  if (!ssm::conv1d_supported(p)) return SSM_ERR_UNSUPPORTED;
  return from_cuda(ssm::launch_conv1d(p, s));
}

ssm_status_t ssm_gated_rmsnorm_fwd(const ssm_gated_norm_args_t *a, void *stream) {
  if (!a) return SSM_ERR_NULL;
  if (a->io != SSM_F32 && a->io != SSM_BF16) return SSM_ERR_DTYPE;
  if (a->rows < 0 || a->width <= 0 || !(a->eps >= 0.f) || a->eps > 3.0e38f) return SSM_ERR_SHAPE;
  if (a->flags) return SSM_ERR_UNSUPPORTED;
  if (a->rows > 0 && (!a->y || !a->out)) return SSM_ERR_NULL;
  if (!all_aligned(a->y, a->z, a->weight, a->out)) return SSM_ERR_ALIGN;
  const size_t bytes = (size_t)a->rows * a->width * (a->io == SSM_BF16 ? 2 : 4);
  auto overlap = [](const void *p, const void *q, size_t n) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p), b0 = reinterpret_cast<uintptr_t>(q);
    return p && q && n > 0 && a0 < b0 + n && b0 < a0 + n;
  };
  // out may be y itself; nothing else may overlap it
  if (a->out != a->y && overlap(a->out, a->y, bytes)) return SSM_ERR_SHAPE;
  if (overlap(a->out, a->z, bytes)) return SSM_ERR_SHAPE;
  ssm::GatedNormParams p;
  p.rows = a->rows;
  p.width = a->width;
  p.io = a->io;
  p.eps = a->eps;
  p.y = a->y;
  p.z = a->z;
  p.weight = a->weight;
  p.out = a->out;
  if (!ssm::gated_norm_supported(p)) return SSM_ERR_UNSUPPORTED;
  if (a->rows == 0) return SSM_OK;
  return from_cuda(ssm::launch_gated_norm(p, static_cast<cudaStream_t>(stream)));
}

namespace {
ssm_status_t check_attn(const ssd_attention_args_t *a, size_t *ws, bool shapes_only) {
  if (!a) return SSM_ERR_NULL;
  if (a->io != SSM_F32 && a->io != SSM_BF16) return SSM_ERR_DTYPE;
  if (a->batch < 0 || a->seqlen < 0 || a->heads <= 0 || a->state <= 0 || a->groups <= 0 ||
      a->heads % a->groups)
    return SSM_ERR_SHAPE;
  if (a->flags & ~SSM_DT_SOFTPLUS) return SSM_ERR_UNSUPPORTED;
  const bool work = a->batch > 0 && a->seqlen > 0;
  if (!shapes_only && work && (!a->dt || !a->B || !a->C || !a->A || !a->alpha))
    return SSM_ERR_NULL;
  if (!shapes_only && !all_aligned(a->dt, a->B, a->C, a->A, a->dt_bias, a->alpha, a->workspace))
    return SSM_ERR_ALIGN;
  ssm::AttnParams p;
  p.batch = a->batch;
  p.L = a->seqlen;
  p.H = a->heads;
  p.N = a->state;
  p.G = a->groups;
  p.heads_per_cta = ssm::attn_heads_per_cta(a->heads, a->groups);
  if (!ssm::attention_supported(p)) return SSM_ERR_UNSUPPORTED;
  *ws = ssm::attention_workspace_bytes(a->batch, a->heads, a->groups, a->seqlen);
  return SSM_OK;
}
}  // namespace

ssm_status_t ssd_attention_workspace(const ssd_attention_args_t *a, size_t *bytes) {
  if (!bytes) return SSM_ERR_NULL;
  size_t ws = 0;
  ssm_status_t st = check_attn(a, &ws, true);
  if (st != SSM_OK) return st;
  *bytes = ws;
  return SSM_OK;
}

ssm_status_t ssd_attention_fwd(const ssd_attention_args_t *a, void *stream) {
  size_t ws = 0;
  ssm_status_t st = check_attn(a, &ws, false);
  if (st != SSM_OK) return st;
  if (a->batch == 0 || a->seqlen == 0) return SSM_OK;
  if (!a->workspace || a->workspace_bytes < ws) return SSM_ERR_WORKSPACE;
  ssm::AttnParams p;
  p.batch = a->batch;
  p.L = a->seqlen;
  p.H = a->heads;
  p.N = a->state;
  p.G = a->groups;
  p.flags = a->flags;
  p.io = a->io;
  p.heads_per_cta = ssm::attn_heads_per_cta(a->heads, a->groups);
  p.dt = a->dt;
  p.B = a->B;
  p.Cm = a->C;
  p.A = a->A;
  p.dt_bias = a->dt_bias;
  p.alpha = a->alpha;
  const size_t nbh = (size_t)(a->batch * a->heads * a->seqlen);
  p.cum = static_cast<double *>(a->workspace);
  p.beta = reinterpret_cast<float *>(static_cast<char *>(a->workspace) + nbh * sizeof(double));
  // C . B^T tiles after the steps, on a 16-byte boundary
  p.cb = reinterpret_cast<float *>(static_cast<char *>(a->workspace) +
                                   ((nbh * (sizeof(double) + sizeof(float)) + 15) & ~(size_t)15));
  p.ntri = ssm::attention_lower_tiles(a->seqlen);
  return from_cuda(ssm::launch_attention(p, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
