// host_pipeline.cu -- ssm_scan_fwd from host buffers (ssm_scan_fwd_host):
// the inputs cross to the GPU, the scan runs, and y, h_last (and the states)
// come back, with the copies in both directions overlapped with each other
// and with the scan.
//
// The batch rows are cut into up to kMaxChunks chunks.  Two slots of device
// buffers in the caller's workspace take turns: chunk i's inputs are copied
// into slot i % 2 on an upload stream while chunk i - 1 is scanned on the
// caller's stream and chunk i - 2's results are copied out on a download
// stream.  Events order each slot's reuse: an upload waits for the scan that
// last read the slot, a scan waits for its upload and for the download of
// the results it is about to overwrite, a download waits for its scan.  The
// host-to-device and device-to-host copies run on separate copy engines, so
// a call takes about the larger of the two directions' copy times instead
// of their sum (the scans, far shorter, hide between them).  The call ends
// with the caller's stream waiting on both copy streams, so that work queued
// after it on that stream (or a synchronize of it) sees every result.
//
// Each chunk is an ordinary scan of its rows (scan_run), the sequence never
// cut when there is more than one chunk, so every (row, channel) is computed
// by the same kernel instance and in the same order as by ssm_scan_fwd on
// the whole batch: the results are bitwise those of the device call.  The
// status word (the workspace's first word) is cleared once, before the first
// chunk, and every chunk's scan reports into it.
//
// The two copy streams and the events are created once per device, on first
// use, and kept for the life of the process; a mutex per device serialises
// the enqueueing of concurrent calls (their GPU work then follows the
// streams' order).
#include <string.h>

#include <mutex>

#include "internal.h"
#include "ssm.h"

namespace {

constexpr int64_t kMaxChunks = 8;
constexpr int kMaxDevices = 64;

size_t r256(size_t v) { return (v + 255) & ~(size_t)255; }

// Offsets in the device workspace.
struct HostPlan {
  int64_t rows = 0, nchunks = 0;  // batch rows per chunk, chunks
  bool cut = false;               // one chunk: the sequence may be cut as usual
  size_t scan_bytes = 0;          // [0, scan_bytes): the scans' workspace
  size_t A = 0, D = 0, dt_bias = 0;
  size_t slot[2] = {0, 0};
  // inside a slot
  size_t x = 0, dt = 0, z = 0, B = 0, C = 0, h0 = 0, y = 0, h_last = 0, states = 0;
  size_t total = 0;
};

HostPlan host_plan(const ssm_scan_args_t *a) {
  HostPlan h;
  const int64_t b = a->batch;
  if (b <= 0) return h;
  h.rows = (b + kMaxChunks - 1) / kMaxChunks;
  h.nchunks = (b + h.rows - 1) / h.rows;
  h.cut = h.nchunks == 1;
  const size_t esz = a->io == SSM_BF16 ? 2 : 4;
  const size_t r = (size_t)h.rows, L = (size_t)a->seqlen, Cn = (size_t)a->channels;
  const size_t N = (size_t)a->state, G = (size_t)a->groups;
  // the scans' workspace: the larger of a whole chunk's and the last one's
  ssm_scan_args_t c = *a;
  c.batch = h.rows;
  size_t ws = ssm::scan_workspace_bytes(&c, h.cut);
  c.batch = b - (h.nchunks - 1) * h.rows;
  const size_t ws_last = ssm::scan_workspace_bytes(&c, h.cut);
  h.scan_bytes = r256(ws > ws_last ? ws : ws_last);
  size_t off = h.scan_bytes;
  h.A = off;
  off += r256(Cn * N * sizeof(float));
  h.D = off;
  off += a->D ? r256(Cn * sizeof(float)) : 0;
  h.dt_bias = off;
  off += a->dt_bias ? r256(Cn * sizeof(float)) : 0;
  size_t s = 0;
  const size_t seq = r256(r * L * Cn * esz), bc = r256(r * L * G * N * esz);
  const size_t state = r256(r * Cn * N * sizeof(float));
  h.x = s;
  s += seq;
  h.dt = s;
  s += seq;
  h.z = s;
  s += a->z ? seq : 0;
  h.B = s;
  s += bc;
  h.C = s;
  s += bc;
  h.h0 = s;
  s += a->h0 ? state : 0;
  h.y = s;
  s += seq;
  h.h_last = s;
  s += a->h_last ? state : 0;
  h.states = s;
  s += a->states ? r256(r * L * Cn * N * sizeof(float)) : 0;
  h.slot[0] = off;
  h.slot[1] = off + s;
  h.total = off + (h.nchunks > 1 ? 2 : 1) * s;  // one chunk needs one slot
  return h;
}

struct Pipeline {
  std::mutex mu;
  bool ready = false;
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t start = nullptr, in[2] = {}, out[2] = {}, freed[2] = {}, up_end = nullptr,
              down_end = nullptr;
};

// The current device's streams and events (created on first use).
Pipeline *pipeline() {
  static Pipeline pipes[kMaxDevices];
  static std::mutex create_mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  Pipeline &p = pipes[dev];
  std::lock_guard<std::mutex> g(create_mu);
  if (p.ready) return &p;
  bool ok = cudaStreamCreateWithFlags(&p.up, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.down, cudaStreamNonBlocking) == cudaSuccess;
  cudaEvent_t *evs[] = {&p.start, &p.in[0], &p.in[1], &p.out[0], &p.out[1],
                        &p.freed[0], &p.freed[1], &p.up_end, &p.down_end};
  for (cudaEvent_t *e : evs)
    ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return nullptr;
  }
  p.ready = true;
  return &p;
}

// Pointer arithmetic on host or device bases.
template <typename T> T *at(T *base, size_t bytes) {
  return reinterpret_cast<T *>(reinterpret_cast<uintptr_t>(base) + bytes);
}
void *dev_at(void *ws, size_t off) { return static_cast<char *>(ws) + off; }

}  // namespace

extern "C" {

ssm_status_t ssm_scan_host_workspace(const ssm_scan_args_t *a, size_t *bytes) {
  if (!bytes) return SSM_ERR_NULL;
  size_t ws = 0;
  const ssm_status_t st = ssm_scan_workspace(a, &ws);  // shapes and flags
  if (st != SSM_OK) return st;
  *bytes = host_plan(a).total;
  return SSM_OK;
}

ssm_status_t ssm_scan_fwd_host(const ssm_scan_args_t *a, void *stream) {
  if (!a) return SSM_ERR_NULL;
  ssm_status_t st = ssm::scan_validate(a);  // every pointer check of ssm_scan_fwd
  if (st != SSM_OK) return st;
  size_t need = 0;
  st = ssm_scan_host_workspace(a, &need);
  if (st != SSM_OK) return st;
  if (a->batch == 0) return SSM_OK;
  if (!a->workspace || a->workspace_bytes < need) return SSM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t esz = a->io == SSM_BF16 ? 2 : 4;
  const int64_t L = a->seqlen, Cn = a->channels, N = a->state, G = a->groups;
  const size_t state_row = (size_t)(Cn * N) * sizeof(float);
  if (cudaMemsetAsync(a->workspace, 0, sizeof(int), s) != cudaSuccess) return SSM_ERR_CUDA;
  if (L == 0) {  // h_last = h0 (or zeros), filled on the host once the stream has drained
    if (!a->h_last) return SSM_OK;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SSM_ERR_CUDA;
    const size_t n = (size_t)a->batch * state_row;
    if (a->h0)
      memcpy(a->h_last, a->h0, n);
    else
      memset(a->h_last, 0, n);
    return SSM_OK;
  }
  Pipeline *pp = pipeline();
  if (!pp) return SSM_ERR_CUDA;
  std::lock_guard<std::mutex> g(pp->mu);
  const HostPlan h = host_plan(a);
  void *ws = a->workspace;
  bool ok = true;
  auto cp = [&](void *dst, const void *src, size_t n, cudaStream_t q) {
    if (ok && n) ok = cudaMemcpyAsync(dst, src, n, cudaMemcpyDefault, q) == cudaSuccess;
  };
  auto rec = [&](cudaEvent_t e, cudaStream_t q) {
    if (ok) ok = cudaEventRecord(e, q) == cudaSuccess;
  };
  auto wait = [&](cudaStream_t q, cudaEvent_t e) {
    if (ok) ok = cudaStreamWaitEvent(q, e, 0) == cudaSuccess;
  };
  // the per-channel constants, once, on the caller's stream; the copy
  // streams start after everything queued there so far
  cp(dev_at(ws, h.A), a->A, (size_t)(Cn * N) * sizeof(float), s);
  if (a->D) cp(dev_at(ws, h.D), a->D, (size_t)Cn * sizeof(float), s);
  if (a->dt_bias) cp(dev_at(ws, h.dt_bias), a->dt_bias, (size_t)Cn * sizeof(float), s);
  rec(pp->start, s);
  wait(pp->up, pp->start);
  wait(pp->down, pp->start);
  ssm_status_t scan_st = SSM_OK;
  for (int64_t i = 0; i < h.nchunks && ok && scan_st == SSM_OK; ++i) {
    const int k = (int)(i & 1);
    const int64_t r0 = i * h.rows, nr = a->batch - r0 < h.rows ? a->batch - r0 : h.rows;
    const size_t seq0 = (size_t)(r0 * L * Cn) * esz, seqn = (size_t)(nr * L * Cn) * esz;
    const size_t bc0 = (size_t)(r0 * L * G * N) * esz, bcn = (size_t)(nr * L * G * N) * esz;
    const size_t st0 = (size_t)r0 * state_row, stn = (size_t)nr * state_row;
    const size_t sq0 = (size_t)(r0 * L) * state_row, sqn = (size_t)(nr * L) * state_row;
    void *slot = dev_at(ws, h.slot[k]);
    // upload: after the scan that last read this slot
    if (i >= 2) wait(pp->up, pp->out[k]);
    cp(dev_at(slot, h.x), at(a->x, seq0), seqn, pp->up);
    cp(dev_at(slot, h.dt), at(a->dt, seq0), seqn, pp->up);
    if (a->z) cp(dev_at(slot, h.z), at(a->z, seq0), seqn, pp->up);
    cp(dev_at(slot, h.B), at(a->B, bc0), bcn, pp->up);
    cp(dev_at(slot, h.C), at(a->C, bc0), bcn, pp->up);
    if (a->h0) cp(dev_at(slot, h.h0), at(a->h0, st0), stn, pp->up);
    rec(pp->in[k], pp->up);
    // the scan: after its upload and the download of this slot's last results
    wait(s, pp->in[k]);
    if (i >= 2) wait(s, pp->freed[k]);
    if (!ok) break;
    ssm_scan_args_t c = *a;
    c.batch = nr;
    c.x = dev_at(slot, h.x);
    c.dt = dev_at(slot, h.dt);
    c.z = a->z ? dev_at(slot, h.z) : nullptr;
    c.B = dev_at(slot, h.B);
    c.C = dev_at(slot, h.C);
    c.A = static_cast<const float *>(dev_at(ws, h.A));
    c.D = a->D ? static_cast<const float *>(dev_at(ws, h.D)) : nullptr;
    c.dt_bias = a->dt_bias ? static_cast<const float *>(dev_at(ws, h.dt_bias)) : nullptr;
    c.h0 = a->h0 ? static_cast<const float *>(dev_at(slot, h.h0)) : nullptr;
    c.y = dev_at(slot, h.y);
    c.h_last = a->h_last ? static_cast<float *>(dev_at(slot, h.h_last)) : nullptr;
    c.states = a->states ? static_cast<float *>(dev_at(slot, h.states)) : nullptr;
    c.workspace = ws;
    c.workspace_bytes = h.scan_bytes;
    scan_st = ssm::scan_run(&c, -1, nullptr, s, h.cut, false);
    if (scan_st != SSM_OK) break;
    rec(pp->out[k], s);
    // download: after the scan
    wait(pp->down, pp->out[k]);
    cp(at(a->y, seq0), c.y, seqn, pp->down);
    if (a->h_last) cp(at(a->h_last, st0), c.h_last, stn, pp->down);
    if (a->states) cp(at(a->states, sq0), c.states, sqn, pp->down);
    rec(pp->freed[k], pp->down);
  }
  // the caller's stream joins both copy streams, whatever happened above
  const bool joined = cudaEventRecord(pp->up_end, pp->up) == cudaSuccess &&
                      cudaEventRecord(pp->down_end, pp->down) == cudaSuccess &&
                      cudaStreamWaitEvent(s, pp->up_end, 0) == cudaSuccess &&
                      cudaStreamWaitEvent(s, pp->down_end, 0) == cudaSuccess;
  if (scan_st != SSM_OK) return scan_st;
  return ok && joined ? SSM_OK : SSM_ERR_CUDA;
}

}  // extern "C"
