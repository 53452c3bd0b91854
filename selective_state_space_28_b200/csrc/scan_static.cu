// scan_static.cu -- ssm_scan_fwd_static: the Mamba-1 scan for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the scan:
// code inside a host framework's enqueue callback that only hands out the
// memory it reserved up front, latency-bound decode loops that must not hit
// an allocator that may synchronise the device, or processes whose device
// memory is fully reserved by another component.  ssm_scan_fwd asks them for
// a workspace (a status word, the step-input RMS factors, and the states of
// sequence segments when it cuts a long sequence).  This entry point takes
// its scratch from a fixed array in the library's own device memory instead:
// the status word and one RMS factor per (batch row, token), with the
// sequence never cut, so the caller passes only its inputs and outputs.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "ssm.h"

namespace {

// Capacity: batch * seqlen RMS factors (1 MiB of float32), after a 256-byte
// status word -- the layout ssm_scan_fwd uses for a workspace without
// segments.
constexpr int64_t kStaticScratchRows = 1 << 18;
constexpr int64_t kStatusFloats = 64;

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) float g_scan_scratch[kStatusFloats + kStaticScratchRows];

// In host code `g_scan_scratch` names a host-side stand-in, not device
// memory: the device address comes from cudaGetSymbolAddress, looked up with
// the device current and cached per device together with the identity of the
// context it was looked up in (a context that is destroyed and recreated,
// e.g. after cudaDeviceReset, may load the module at another address, so a
// changed context id forces a new lookup).
constexpr int kMaxDevices = 64;
struct Entry {
  unsigned long long ctx_id = 0;
  void *addr = nullptr;
};
Entry g_cache[kMaxDevices];
std::mutex g_mu;

// The current context's id, or 0 when the driver entry points are missing.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static bool looked = false;
  if (!looked) {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    looked = true;
  }
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace

namespace ssm {

cudaError_t static_scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long id = current_context_id();
  if (id != 0 && g_cache[dev].addr && g_cache[dev].ctx_id == id) {
    *out = g_cache[dev].addr;
    return cudaSuccess;
  }
  void *p = nullptr;
  e = cudaGetSymbolAddress(&p, g_scan_scratch);
  if (e != cudaSuccess) return e;
  g_cache[dev].addr = p;
  g_cache[dev].ctx_id = current_context_id();  // the lookup may have created the context
  *out = p;
  return cudaSuccess;
}

}  // namespace ssm

extern "C" ssm_status_t ssm_scan_fwd_static(const ssm_scan_args_t *args, void *stream) {
  if (!args) return SSM_ERR_NULL;
  // Every host-side check first: nothing touches the device for a bad call.
  ssm_scan_args_t a = *args;
  a.workspace = nullptr;
  a.workspace_bytes = 0;
  const ssm_status_t st = ssm::scan_validate(&a);
  if (st != SSM_OK) return st;
  if (a.batch == 0) return SSM_OK;  // nothing to do, nothing launched
  // Reject problems the scratch cannot hold.
  if ((a.flags & SSM_RMSNORM_DT) && a.batch > 0 && a.seqlen > 0 &&
      a.batch > kStaticScratchRows / a.seqlen)
    return SSM_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (ssm::static_scratch_address(&scratch) != cudaSuccess) return SSM_ERR_CUDA;
  // Same kernels as ssm_scan_fwd, the sequence never cut.  The status word is
  // cleared by every call; the RMS factors need no clearing (the pre-pass
  // writes every one the scan reads).
  a.workspace = scratch;
  a.workspace_bytes = sizeof(g_scan_scratch);
  return ssm::scan_run(&a, -1, nullptr, stream, false);
}
