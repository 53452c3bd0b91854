/*
 * ssm.h -- C ABI of libssm: the selective state-space scan on NVIDIA B200
 * (sm_100a).
 *
 * Three operations, each a plain C call on plain pointers and sizes:
 *
 *   ssm_scan_fwd        Mamba-1 selective scan over a prompt
 *                       (ssm_scan_fwd_write: with a state written at one token).
 *   ssd_chunk_scan_fwd  Mamba-2 (SSD) scan over a prompt, chunked
 *                       (ssd_conv_chunk_scan_fwd: with the mixer's causal
 *                       convolution fused in front of it).
 *   ssm_scan_step       one decode token against a cached state.
 *   ssm_conv1d_fwd      the mixers' causal depthwise convolution (+ silu),
 *                       over a prompt or, in place, one decode token.
 *   ssm_gated_rmsnorm_fwd  the Mamba-2 mixer's gated RMS norm after the SSD.
 *   ssd_attention_fwd   the SSD map's hidden attention matrix, per head.
 *
 * Conventions for every call
 * --------------------------
 * - Pointers are DEVICE pointers (cudaMalloc'd or otherwise device-visible),
 *   owned by the caller.  The library allocates nothing, keeps no state
 *   between calls, and is reentrant.  Work is queued on `stream` (a
 *   cudaStream_t passed as void*; NULL = the legacy default stream) and the
 *   call returns without synchronising; results are ordered on `stream`.
 * - Layouts are dense, row-major and tokens-first, as the pages' values are
 *   ("Mamba" nnterp guide, "The values" table: x is [batch, seq, channels],
 *   state is [batch, channels, state_dim]; "Mamba-2": the state is
 *   [batch, heads, key_dim, value_dim], key side first).
 * - `io` selects the element type of x, dt, z, B, C and y (SSM_F32 or
 *   SSM_BF16).  A, D, dt_bias and every state are float32, and all
 *   arithmetic is float32.
 * - Arguments are validated on the host before anything is launched.  On an
 *   error the call returns a status and launches nothing.  Launch failures
 *   return SSM_ERR_CUDA.  There is no CPU fallback.
 * - Aliasing: inputs and outputs must not overlap, except that h_last may
 *   equal h0 (the state hand-off), and the decode step updates its state in
 *   place.
 */
#ifndef SSM_H
#define SSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSM_ABI_VERSION 4

typedef enum ssm_status {
  SSM_OK = 0,
  SSM_ERR_NULL = 1,        /* a required pointer is NULL                      */
  SSM_ERR_SHAPE = 2,       /* a size is <= 0, or groups does not divide       */
  SSM_ERR_DTYPE = 3,       /* io is not SSM_F32 / SSM_BF16                    */
  SSM_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned                */
  SSM_ERR_UNSUPPORTED = 5, /* a valid combination the library has no kernel for */
  SSM_ERR_WORKSPACE = 6,   /* workspace missing or smaller than required      */
  SSM_ERR_CUDA = 7,        /* a CUDA launch or runtime call failed            */
  SSM_ERR_TIMEOUT = 8      /* a bounded device wait ran out (see
                              ssm_workspace_status)                           */
} ssm_status_t;

typedef enum ssm_dtype { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype_t;

/* flags */
#define SSM_DT_SOFTPLUS 1u /* step = softplus(dt + dt_bias); else dt + dt_bias  */
#define SSM_RMSNORM_BC 2u  /* B, C <- v / sqrt(mean_N(v^2) + rms_eps) (no gain) */
#define SSM_RMSNORM_DT 4u  /* dt <- dt / sqrt(mean_C(dt^2) + rms_eps), before
                              the bias (Mamba-1 scan only)                      */

/* ------------------------------------------------------------------------
 * ssm_scan_fwd -- Mamba-1 selective scan.
 *
 * Defined by: "Mamba" (nnterp guide, architectures/mamba), intro and "The
 * values" table; "Mamba" (tokentrails lineage), "Code"; "Falcon-Mamba"
 * (nnterp encyclopedia), "Where the norms sit" for the two RMS flags.
 * For every batch b, channel c (group g = c / (channels / groups)) and token t:
 *
 *   d     = dt[b,t,c]  (* RMS factor of dt[b,t,:] if SSM_RMSNORM_DT)
 *   d     = softplus(d + dt_bias[c])  (or d + dt_bias[c] without SSM_DT_SOFTPLUS)
 *   h[n]  = exp(d * A[c,n]) * h[n] + d * B[b,t,g,n] * x[b,t,c]   (n < state)
 *   y     = sum_n C[b,t,g,n] * h[n] + D[c] * x[b,t,c]
 *   y    *= silu(z[b,t,c])             if z != NULL
 *
 * with h starting from h0[b,c,:] (zeros if h0 == NULL).  y_t reads the state
 * after token t's write.
 *
 *   x, dt, z, y : [batch, seqlen, channels]   io type; z may be NULL (no gate)
 *   B, C        : [batch, seqlen, groups, state]  io type
 *   A           : [channels, state]  float32 (pass -exp(A_log))
 *   D, dt_bias  : [channels]         float32, may be NULL (= 0)
 *   h0          : [batch, channels, state] float32 or NULL (= zeros)
 *   h_last      : [batch, channels, state] float32 or NULL; may equal h0
 *   states      : [batch, seqlen, channels, state] float32 or NULL: the state
 *                 after every token (states[:, -1] == h_last bit for bit)
 *   workspace   : device memory of ssm_scan_workspace() bytes (at least 256),
 *                 caller-owned.  Word 0 (int32) is the call's status word:
 *                 the call zeroes it, and a kernel whose bounded wait for its
 *                 own copies runs out (about a second: a fault elsewhere on the
 *                 device) sets it non-zero and leaves y and h_last
 *                 incomplete; ssm_workspace_status() reads it.  The rest
 *                 holds the step-input RMS factors (SSM_RMSNORM_DT) and, when
 *                 batch x channels is too small to fill the device's SMs,
 *                 the states of the sequence segments the scan is cut into
 *                 (their end states, the sums of their steps and the carried
 *                 states); its size therefore depends on the device current at
 *                 the query, and a call with less than its own device needs
 *                 returns SSM_ERR_WORKSPACE.
 *
 * Supported: state in {4, 8, 16, 32, 64}; groups must divide channels, and
 * with groups > 1 channels/groups must be a multiple of 32.
 * ---------------------------------------------------------------------- */
typedef struct ssm_scan_args {
  int64_t batch, seqlen, channels, state, groups;
  int32_t io;        /* ssm_dtype_t */
  uint32_t flags;
  float rms_eps;
  const void *x, *dt, *z, *B, *C;
  const float *A, *D, *dt_bias, *h0;
  void *y;
  float *h_last, *states;
  void *workspace;
  size_t workspace_bytes;
} ssm_scan_args_t;

/* Bytes of device workspace ssm_scan_fwd needs for these arguments.
 * Validates sizes, dtype and flags as ssm_scan_fwd does; the tensor pointers
 * are not looked at. */
ssm_status_t ssm_scan_workspace(const ssm_scan_args_t *args, size_t *bytes);
ssm_status_t ssm_scan_fwd(const ssm_scan_args_t *args, void *stream);

/* ssm_scan_fwd_static -- ssm_scan_fwd without a caller-provided workspace.
 *
 * The pages have no counterpart: this is a deployment variant.  Some callers
 * cannot allocate device memory where they run the scan -- an engine's
 * enqueue callback that may only use memory reserved up front, a decode loop
 * with a latency budget that must not meet an allocator that can
 * synchronise the device, a process whose device memory another component
 * has reserved.  ssm_scan_fwd needs a caller workspace (a status word, the
 * step-input RMS factors with SSM_RMSNORM_DT, and sequence segments' states
 * when it cuts a long sequence); this entry point uses a fixed array in the
 * library's own device memory instead (static, 256 bytes + 1 MiB per GPU,
 * held until the process exits) and never cuts the sequence, so the caller
 * passes only inputs and outputs.
 *
 * Arguments, layouts, results and errors are those of ssm_scan_fwd;
 * args->workspace is ignored.  Every host-side check runs before anything
 * touches the device.  Limit: with SSM_RMSNORM_DT, batch * seqlen must not
 * exceed 262144; larger problems return SSM_ERR_WORKSPACE.  The first call
 * on each device (and after the device's context is recreated) looks up the
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  All calls share the
 * array, which keeps the last call's contents: each call clears the status
 * word it uses, and the RMS factors need no clearing (every one the scan
 * reads is written first).  Calls that overlap on the GPU -- on different
 * streams, or from several threads -- race on it and must be serialised by
 * the caller.  ssm_workspace_status(NULL, stream) reads its status word. */
ssm_status_t ssm_scan_fwd_static(const ssm_scan_args_t *args, void *stream);

/* ssm_scan_fwd_host -- ssm_scan_fwd for a caller whose tensors live in HOST
 * memory.
 *
 * The pages have no counterpart: this is the end-to-end form of the same
 * scan.  x, dt, z, B, C, A, D, dt_bias, h0 are host pointers to the inputs,
 * y, h_last (and states, when not NULL) host pointers that receive the
 * results, all in ssm_scan_fwd's layouts; args->workspace is DEVICE memory
 * of ssm_scan_host_workspace() bytes (two chunks' device copies of the
 * inputs and results, the per-channel constants and the scan's own
 * workspace; its first word is the status word, as for ssm_scan_fwd).
 *
 * The batch rows are taken in up to 8 chunks: while one chunk is scanned on
 * `stream`, the next chunk's inputs are copied in and the previous chunk's
 * results copied out on two streams of the library's own (created once per
 * device, on first use), so that the two directions' copies overlap each
 * other and the scans; `stream` waits for both copy streams before the call
 * returns, so a synchronize of `stream` (or work queued on it after the
 * call) sees every result.  With page-locked (pinned) host buffers the call
 * only enqueues; pageable buffers work too, but the runtime then copies them
 * synchronously and nothing overlaps.  The caller must leave the inputs
 * unchanged and not read the outputs until `stream` has completed the call.
 * Results are bitwise those of ssm_scan_fwd on the same inputs (every chunk
 * runs the same kernels on its rows; the sequence is never cut into
 * segments when there is more than one chunk).  With seqlen 0 the call
 * synchronises `stream` and fills h_last from h0 (or zeros) on the host.
 * Calls from several threads are enqueued one at a time (a lock per device);
 * each needs its own workspace.  Errors: those of ssm_scan_fwd, checked
 * before anything is enqueued; SSM_ERR_CUDA when a copy or an event cannot
 * be enqueued (stream then still waits for what was enqueued). */
ssm_status_t ssm_scan_host_workspace(const ssm_scan_args_t *args, size_t *bytes);
ssm_status_t ssm_scan_fwd_host(const ssm_scan_args_t *args, void *stream);

/* ssm_scan_fwd_write -- ssm_scan_fwd with the state written at one token.
 *
 * Defined by: "Mamba" (nnterp guide), "The state": writing the state at
 * token t replaces h_t -- y_t reads the written state (a write at token t
 * changes token t's own output) and tokens t+1.. continue from it.
 * state_write: [batch, channels, state] float32, 0 <= t_write < seqlen.
 * Everything else as ssm_scan_fwd (same workspace query).  (The Mamba-2
 * page marks the same write unavailable for the chunked scan: there is no
 * SSD counterpart.) */
ssm_status_t ssm_scan_fwd_write(const ssm_scan_args_t *args, int64_t t_write,
                                const float *state_write, void *stream);

/* ssm_workspace_status -- did the call that used this workspace finish?
 *
 * Synchronises `stream`, reads word 0 of `workspace` (a workspace of
 * ssm_scan_fwd, ssm_scan_fwd_write or ssd_chunk_scan_fwd, after a call queued
 * on `stream`) and returns SSM_OK, or SSM_ERR_TIMEOUT when one of that call's
 * bounded device waits ran out (its outputs are then incomplete).
 * workspace == NULL reads the status word of ssm_scan_fwd_static's static
 * scratch on the current device.  SSM_ERR_CUDA if the copy or the
 * synchronisation fails. */
ssm_status_t ssm_workspace_status(const void *workspace, void *stream);

/* ------------------------------------------------------------------------
 * ssd_chunk_scan_fwd -- Mamba-2 (SSD) scan.
 *
 * Defined by: "Mamba-2" (nnterp encyclopedia), "The mixer's values" (one
 * scalar decay per head and token; B and C shared by the heads of a group),
 * "The hidden attention" (the causal masked form the chunked algorithm
 * evaluates), "The state" (key side first).  For batch b, head h (group
 * g = h / (heads / groups)), token t:
 *
 *   d      = softplus(dt[b,t,h] + dt_bias[h])   (flag SSM_DT_SOFTPLUS)
 *   S      = exp(d * A[h]) * S + d * outer(B[b,t,g,:], x[b,t,h,:])   (N x P)
 *   y[p]   = sum_n C[b,t,g,n] * S[n,p] + D[h] * x[b,t,h,p];  *= silu(z) if z
 *
 * evaluated chunk by chunk (`chunk` tokens): within a chunk as the masked
 * product y_t = sum_{s<=t} (C_t . B_s) exp(cum_t - cum_s) d_s x_s, across
 * chunks through the carried N x P state.  The result does not depend on
 * `chunk` beyond rounding.
 *
 *   x, z, y  : [batch, seqlen, heads, head_dim]  io type; z may be NULL
 *   dt       : [batch, seqlen, heads]            io type
 *   B, C     : [batch, seqlen, groups, state]    io type
 *   A        : [heads] float32; D, dt_bias: [heads] float32 or NULL (= 0)
 *   h0       : [batch, heads, state, head_dim] float32 or NULL (= zeros)
 *   h_last   : [batch, heads, state, head_dim] float32 or NULL; may equal h0
 *   states   : [batch, seqlen, heads, state, head_dim] float32 or NULL
 *   workspace: device memory of ssd_chunk_scan_workspace() bytes, or NULL if
 *              that is 0.  When non-zero, word 0 (int32) is the call's
 *              status word, as for ssm_scan_fwd: zeroed by the call, set
 *              non-zero when a bounded device wait runs out (y and h_last
 *              then incomplete); read it with ssm_workspace_status().
 *
 * Only SSM_DT_SOFTPLUS is accepted in flags.
 * ---------------------------------------------------------------------- */
typedef struct ssd_scan_args {
  int64_t batch, seqlen, heads, head_dim, state, groups, chunk;
  int32_t io;
  uint32_t flags;
  const void *x, *z, *dt, *B, *C;
  const float *A, *D, *dt_bias, *h0;
  void *y;
  float *h_last, *states;
  void *workspace;
  size_t workspace_bytes;
} ssd_scan_args_t;

/* Bytes of device workspace ssd_chunk_scan_fwd needs (sizes, dtype and flags
 * are validated; the tensor pointers are not looked at).  On the tensor-core
 * path (bf16, state 128, head_dim 64, no per-token states) it holds a status
 * word and, when batch x heads leaves the last wave of the current device's
 * SMs partial, the float32 end states, carried states and decay products of
 * the sequence segments that wave is cut into; the size therefore depends on
 * the device current at the query (148 SMs are assumed when none can be
 * read), and a call with less workspace than its own device needs returns
 * SSM_ERR_WORKSPACE. */
ssm_status_t ssd_chunk_scan_workspace(const ssd_scan_args_t *args, size_t *bytes);
ssm_status_t ssd_chunk_scan_fwd(const ssd_scan_args_t *args, void *stream);

/* ------------------------------------------------------------------------
 * ssd_conv_chunk_scan_fwd -- the Mamba-2 mixer's causal convolution and the
 * SSD scan in one call.
 *
 * Defined by: "Mamba-2" (nnterp encyclopedia), the module tree
 * (Conv1d(channels, channels, kernel_size 4, padding 3, groups = channels),
 * output cut to the input length) and "The mixer's values" (x, B, C =
 * silu(conv1d(xBC)) split by channel, then the SSD).  With
 * channels = heads * head_dim + 2 * groups * state:
 *
 *   u[t, c] = silu(conv_bias[c] + sum_{k<4} conv_w[c, k] * xBC[t - 3 + k, c])
 *   x = u[.., 0 : heads*head_dim] as [.., heads, head_dim],
 *   B = the next groups*state channels, C = the last groups*state,
 *   then y and h_last exactly as ssd_chunk_scan_fwd computes them.
 *
 *   xBC            : [batch, seqlen, channels] bf16, before the convolution
 *   conv_w         : [channels, 4] float32; conv_bias: [channels] or NULL (0)
 *   conv_state_in  : [batch, channels, 3] float32 or NULL (zeros, a sequence
 *                    start): the inputs of the 3 tokens before t = 0,
 *                    oldest first
 *   conv_state_out : [batch, channels, 3] float32 or NULL: the last 3
 *                    inputs (conv_state_in's entries where seqlen < 3), so a
 *                    prompt cut in two and run with conv_state_out ->
 *                    conv_state_in gives the same y; must not overlap
 *                    conv_state_in (SSM_ERR_SHAPE)
 *   z, dt, A, D, dt_bias, h0, y, h_last, chunk, flags: as ssd_chunk_scan_fwd
 *   workspace      : ssd_conv_chunk_scan_workspace() bytes: the status word
 *                    (word 0, read with ssm_workspace_status()), the
 *                    convolved B and C (batch * seqlen * 2 * groups * state
 *                    bf16) and the segment states of a cut last wave (as
 *                    for ssd_chunk_scan_fwd; device-dependent size)
 *
 * The convolved x is never written to memory: each 128-token tile of x is
 * convolved in shared memory where it lands; B and C, which every head of a
 * group reads, are convolved once by a pre-pass.  bf16 silu as
 * ssm_conv1d_fwd.  Only the tensor-core configuration is taken (io
 * SSM_BF16, state 128, head_dim 64; else SSM_ERR_UNSUPPORTED: run
 * ssm_conv1d_fwd then ssd_chunk_scan_fwd).
 * ---------------------------------------------------------------------- */
typedef struct ssd_conv_scan_args {
  int64_t batch, seqlen, heads, head_dim, state, groups, chunk;
  int32_t io;
  uint32_t flags;
  const void *xBC;
  const float *conv_w, *conv_bias, *conv_state_in;
  float *conv_state_out;
  const void *z, *dt;
  const float *A, *D, *dt_bias, *h0;
  void *y;
  float *h_last;
  void *workspace;
  size_t workspace_bytes;
} ssd_conv_scan_args_t;

ssm_status_t ssd_conv_chunk_scan_workspace(const ssd_conv_scan_args_t *args, size_t *bytes);
ssm_status_t ssd_conv_chunk_scan_fwd(const ssd_conv_scan_args_t *args, void *stream);

/* ------------------------------------------------------------------------
 * ssm_scan_step -- one decode token per sequence, state updated in place.
 *
 * Defined by: "Mamba" (nnterp guide), "The state" and the "Read order on a
 * decode step" warning: the decode kernel updates the state first and reads
 * y from the updated state; the state is handed from one step's output to
 * the next step's input.  "Mamba-2", "The state", for the N x P form.
 *
 * SSM_STEP_MAMBA1: units = channels, head_dim = 1.
 *   x, dt, z, y: [batch, channels]; B, C: [batch, groups, state];
 *   A: [channels, state]; D, dt_bias: [channels]; state: [batch, channels, state]
 * SSM_STEP_MAMBA2: units = heads.
 *   x, z, y: [batch, heads, head_dim]; dt: [batch, heads];
 *   B, C: [batch, groups, state]; A, D, dt_bias: [heads];
 *   state: [batch, heads, state, head_dim] (key side first)
 *
 * The arithmetic is one token of ssm_scan_fwd / ssd_chunk_scan_fwd.  flags:
 * SSM_DT_SOFTPLUS, and for Mamba-1 also SSM_RMSNORM_BC.
 * ---------------------------------------------------------------------- */
typedef enum ssm_step_kind { SSM_STEP_MAMBA1 = 1, SSM_STEP_MAMBA2 = 2 } ssm_step_kind_t;

typedef struct ssm_step_args {
  int32_t kind; /* ssm_step_kind_t */
  int32_t io;
  uint32_t flags;
  float rms_eps;
  int64_t batch, units, head_dim, state, groups;
  const void *x, *dt, *z, *B, *C;
  const float *A, *D, *dt_bias;
  float *state_io;
  void *y;
} ssm_step_args_t;

ssm_status_t ssm_scan_step(const ssm_step_args_t *args, void *stream);

/* ------------------------------------------------------------------------
 * ssm_conv1d_fwd -- the mixers' causal depthwise convolution, then silu.
 *
 * Defined by: "Mamba-2" (nnterp encyclopedia), the module tree
 * (Conv1d(channels, channels, kernel_size 4, padding 3, groups = channels))
 * and "The mixer's values" (x, B, C = silu(conv1d(xBC)), causal, width 4);
 * "Mamba" (tokentrails lineage), "Code" (x = silu(causal_conv1d(x)),
 * depthwise, width 4).  The layer's output is cut to the input length, so
 *
 *   u[t, c] = act(bias[c] + sum_{k < width} w[c, k] * x[t - (width - 1) + k, c])
 *
 * with act = silu when flags has SSM_CONV_SILU, else the identity.
 *   x, u: [batch, seqlen, channels] (io); w: [channels, width] float32;
 *   bias: [channels] float32 or NULL (zero);
 *   state_in: [batch, channels, width - 1] float32 or NULL (zeros, a
 *     sequence start): the inputs of the width - 1 tokens before t = 0,
 *     oldest first;
 *   state_out: [batch, channels, width - 1] float32 or NULL: the last
 *     width - 1 inputs (state_in's entries where seqlen < width - 1), so a
 *     sequence cut in two and run with state_out -> state_in gives the same
 *     u.
 * width 1..4 (else SSM_ERR_UNSUPPORTED).  state_out may equal state_in:
 * with seqlen 1 that is the decode form (state updated in place); no other
 * overlap is allowed, and x and u must not overlap.  seqlen 0 copies (or
 * zeroes) the state.  bf16 outputs use silu = z (1 + tanh(z / 2)) / 2 with
 * the hardware tanh; float32 uses z / (1 + exp(-z)).
 * ---------------------------------------------------------------------- */
#define SSM_CONV_SILU 1u

typedef struct ssm_conv_args {
  int64_t batch, seqlen, channels, width;
  int32_t io;
  uint32_t flags;
  const void *x;
  const float *w, *bias, *state_in;
  void *u;
  float *state_out;
} ssm_conv_args_t;

ssm_status_t ssm_conv1d_fwd(const ssm_conv_args_t *args, void *stream);

/* ------------------------------------------------------------------------
 * ssm_gated_rmsnorm_fwd -- the Mamba-2 mixer's gated norm, after the SSD.
 *
 * Defined by: "Mamba-2" (nnterp encyclopedia), "The mixer's values"
 * (return out_proj(norm(y * silu(z)))) and the paragraph on the block's
 * norms: the gated norm multiplies y by silu(z) and then normalizes over the
 * mixer's whole width, whatever n_groups is.  Per row (one token's
 * heads x head_dim values):
 *
 *   g = y * silu(z)   (g = y when z is NULL)
 *   out = g / sqrt(mean(g^2) + eps) * weight   (weight NULL = ones)
 *
 *   y, z, out: [rows, width] (io); weight: [width] float32.
 * rows = batch * seqlen tokens, width 1..49152.  out may equal y (in place);
 * no other overlap.  flags must be 0.  bf16 uses silu = z (1 + tanh(z/2)) / 2
 * with the hardware tanh; float32 uses z / (1 + exp(-z)).
 * ---------------------------------------------------------------------- */
typedef struct ssm_gated_norm_args {
  int64_t rows, width;
  int32_t io;
  uint32_t flags;
  float eps;
  const void *y, *z;
  const float *weight;
  void *out;
} ssm_gated_norm_args_t;

ssm_status_t ssm_gated_rmsnorm_fwd(const ssm_gated_norm_args_t *args, void *stream);

/* ------------------------------------------------------------------------
 * ssd_attention_fwd -- the hidden attention of the Mamba-2 (SSD) map.
 *
 * Defined by: "Mamba-2" (nnterp encyclopedia), "The hidden attention": per
 * head the scan is a causal linear map over tokens, y_t = sum_s
 * alpha[t, s] x_s + D x_t (zero initial state), with
 *
 *   alpha[t, s] = (C_t . B_s) * exp(decays_{s+1} + ... + decays_t) * betas_s
 *
 * for s <= t and 0 above the diagonal; betas = softplus(dt + dt_bias) when
 * flags has SSM_DT_SOFTPLUS (else dt + dt_bias), decays = betas * A_h, and
 * head h reads group h / (heads / groups).
 *   dt: [batch, seqlen, heads] (io); B, C: [batch, seqlen, groups, state]
 *   (io); A, dt_bias: [heads] float32 (dt_bias may be NULL);
 *   alpha: [batch, heads, seqlen, seqlen] float32 (query t, key s), every
 *   entry written.
 * state 1..256.  The workspace (ssd_attention_workspace) holds the steps and
 * the running decay sums (float64).  The decay factor is exact for A <= 0
 * (a decaying state); it is taken as a product of two factors below the
 * diagonal 32 x 32 blocks, each <= 1 in that case.
 * ---------------------------------------------------------------------- */
typedef struct ssd_attention_args {
  int64_t batch, seqlen, heads, state, groups;
  int32_t io;
  uint32_t flags;
  const void *dt, *B, *C;
  const float *A, *dt_bias;
  float *alpha;
  void *workspace;
  size_t workspace_bytes;
} ssd_attention_args_t;

ssm_status_t ssd_attention_workspace(const ssd_attention_args_t *args, size_t *bytes);
ssm_status_t ssd_attention_fwd(const ssd_attention_args_t *args, void *stream);

/* A short English description of a status; never NULL. */
const char *ssm_status_string(ssm_status_t status);
/* SSM_ABI_VERSION of the library. */
int ssm_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SSM_H */
