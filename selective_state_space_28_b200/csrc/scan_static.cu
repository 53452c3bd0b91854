// scan_static.cu -- ssm_scan_fwd_static: the Mamba-1 scan for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the scan:
// code inside a host framework's enqueue callback that only hands out the
// memory it reserved up front, latency-bound decode loops that must not hit
// an allocator that may synchronise the device, or processes whose device
// memory is fully reserved by another component.  ssm_scan_fwd asks them for
// a workspace whenever the step-input RMS norm is on (one float per batch row
// and token).  This entry point takes that scratch from a fixed array in the
// library's own device memory instead, so the caller passes only its inputs
// and outputs.
#include <atomic>

#include <cuda_runtime.h>

#include "ssm.h"

namespace {

// Capacity of the scratch: batch * seqlen RMS factors (1 MiB of float32).
constexpr int64_t kStaticScratchRows = 1 << 18;

// One float per (batch row, token).  Every GPU that loads the library holds
// this array until the process exits.
static __device__ __align__(256) float g_scan_scratch[kStaticScratchRows];

// In host code `g_scan_scratch` names a host-side stand-in, not device
// memory: the device address comes from cudaGetSymbolAddress, looked up once
// per device with that device current, and cached here.
constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];

cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_scan_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" ssm_status_t ssm_scan_fwd_static(const ssm_scan_args_t *args, void *stream) {
  if (!args) return SSM_ERR_NULL;
  // Reject problems the scratch cannot hold before touching the device.
  if ((args->flags & SSM_RMSNORM_DT) && args->batch > 0 && args->seqlen > 0 &&
      args->batch > kStaticScratchRows / args->seqlen)
    return SSM_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return SSM_ERR_CUDA;
  // Same validation and kernels as ssm_scan_fwd; only the workspace differs.
  // No factor needs clearing: the pre-pass writes every one the scan reads.
  ssm_scan_args_t a = *args;
  a.workspace = scratch;
  a.workspace_bytes = (size_t)kStaticScratchRows * sizeof(float);
  return ssm_scan_fwd(&a, stream);
}
