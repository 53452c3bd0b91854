/*
 * ssm_oracle.h -- float64 CPU oracle for the selective state-space scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this code: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * Every array is a dense, row-major float64 array.  Optional inputs may be
 * NULL (D, dt_bias, h0 -> zeros; z -> no gate); optional outputs may be NULL.
 *
 * Sources (page title, section):
 *   - "Mamba" (nnterp guide, architectures/mamba): intro paragraph (the
 *     per-channel recurrence), "The values" table (layouts, betas =
 *     softplus(dt + dt_bias), y = C.h + D*x before the gate), "The state"
 *     (state after every token, decode step updates first then reads).
 *   - "Mamba" (tokentrails lineage), "Code" and steps 3-4.
 *   - "Mamba-2" (nnterp encyclopedia), "The mixer's values", "The hidden
 *     attention", "The state", "A zero step skips a token exactly".
 *   - "Falcon-Mamba" (nnterp encyclopedia), "Where the norms sit".
 *   - The mixers' causal convolution: "Mamba-2" (nnterp encyclopedia), the
 *     module tree (Conv1d, kernel 4, padding 3, groups = channels) and "The
 *     mixer's values" (x, B, C = silu(conv1d(xBC)), causal, width 4);
 *     "Mamba" (tokentrails lineage), "Code" (x = silu(causal_conv1d(x)),
 *     depthwise, width 4).
 *   - The Mamba-2 mixer's gated norm: "Mamba-2" (nnterp encyclopedia), "The
 *     mixer's values" (out_proj(norm(y * silu(z)))) and the paragraph on the
 *     block's norms (the gated norm multiplies y by silu(z), then normalizes
 *     over the mixer's whole width, whatever n_groups is).
 */
#ifndef SSM_ORACLE_H
#define SSM_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_SOFTPLUS 1u  /* dt <- softplus(dt + dt_bias)                     */
#define ORC_RMS_BC   2u  /* B, C <- weightless RMS norm over the state axis   */
#define ORC_RMS_DT   4u  /* dt_raw <- weightless RMS norm over the channels   */

/* Mamba-1 selective scan.  x, dt, z, y: [b, L, C]; B, Cm: [b, L, G, N];
 * A: [C, N]; D, dt_bias: [C]; h0, h_last: [b, C, N]; states: [b, L, C, N].
 * Channel c reads group c / (C / G).  Work is split over nthreads threads. */
int orc_m1_scan(int64_t batch, int64_t seqlen, int64_t channels, int64_t state,
                int64_t groups, uint32_t flags, double rms_eps,
                const double *x, const double *dt, const double *z,
                const double *B, const double *Cm, const double *A,
                const double *D, const double *dt_bias, const double *h0,
                double *y, double *h_last, double *states, int nthreads);

/* orc_m1_scan with a state written at token t_write ("Mamba", nnterp guide,
 * "The state": writing the state at token t replaces h_t, so y_t reads the
 * written state and tokens t+1.. continue from it).  state_write: [b, C, N];
 * 0 <= t_write < seqlen. */
int orc_m1_scan_write(int64_t batch, int64_t seqlen, int64_t channels, int64_t state,
                      int64_t groups, uint32_t flags, double rms_eps,
                      const double *x, const double *dt, const double *z,
                      const double *B, const double *Cm, const double *A,
                      const double *D, const double *dt_bias, const double *h0,
                      int64_t t_write, const double *state_write,
                      double *y, double *h_last, double *states, int nthreads);

/* Mamba-2 (SSD) scan, written as the token recurrence.  x, z, y: [b, L, H, P];
 * dt: [b, L, H]; B, Cm: [b, L, G, N]; A, D, dt_bias: [H];
 * h0, h_last: [b, H, N, P] (key side first); states: [b, L, H, N, P].
 * Head h reads group h / (H / G).  Only ORC_SOFTPLUS is meaningful. */
int orc_m2_scan(int64_t batch, int64_t seqlen, int64_t heads, int64_t head_dim,
                int64_t state, int64_t groups, uint32_t flags,
                const double *x, const double *dt, const double *z,
                const double *B, const double *Cm, const double *A,
                const double *D, const double *dt_bias, const double *h0,
                double *y, double *h_last, double *states, int nthreads);

/* One decode token, Mamba-1: state [b, C, N] is updated in place, then read.
 * x, dt, z, y: [b, C]; B, Cm: [b, G, N]. */
int orc_m1_step(int64_t batch, int64_t channels, int64_t state, int64_t groups,
                uint32_t flags, double rms_eps,
                const double *x, const double *dt, const double *z,
                const double *B, const double *Cm, const double *A,
                const double *D, const double *dt_bias,
                double *state_io, double *y);

/* One decode token, Mamba-2: state [b, H, N, P] updated in place, then read.
 * x, z, y: [b, H, P]; dt: [b, H]; B, Cm: [b, G, N]. */
int orc_m2_step(int64_t batch, int64_t heads, int64_t head_dim, int64_t state,
                int64_t groups, uint32_t flags,
                const double *x, const double *dt, const double *z,
                const double *B, const double *Cm, const double *A,
                const double *D, const double *dt_bias,
                double *state_io, double *y);

/* Brute-force quadratic ("hidden attention") form, Mamba-2 layout, O(L^3):
 *   y_t = sum_{s<=t} (C_t . B_s) * exp(sum_{r=s+1..t} dt_r A) * dt_s * x_s
 *         + C_t . (exp(sum_{r<=t} dt_r A) h0) + D x_t,   then the gate.
 * dt here is the step AFTER bias and softplus (the pages' "betas"). */
int orc_m2_quadratic(int64_t batch, int64_t seqlen, int64_t heads,
                     int64_t head_dim, int64_t state, int64_t groups,
                     const double *x, const double *betas, const double *z,
                     const double *B, const double *Cm, const double *A,
                     const double *D, const double *h0, double *y);

/* The same quadratic form for Mamba-1 (per channel c and state n, A[c, n]).
 * betas: [b, L, C], the step after bias/softplus; B, Cm already normed. */
int orc_m1_quadratic(int64_t batch, int64_t seqlen, int64_t channels,
                     int64_t state, int64_t groups,
                     const double *x, const double *betas, const double *z,
                     const double *B, const double *Cm, const double *A,
                     const double *D, const double *h0, double *y);

/* Causal depthwise convolution over tokens, then silu when act != 0: the
 * module tree's Conv1d(channels, channels, kernel W, padding W - 1,
 * groups = channels) with its output cut to the input length, so
 *   u[t, c] = bias[c] + sum_{k<W} w[c, k] * x[t - (W - 1) + k, c].
 * x, u: [b, L, Cc]; w: [Cc, W]; bias: [Cc] or NULL (zero); state_in:
 * [b, Cc, W - 1], the inputs of the W - 1 tokens before t = 0, oldest first,
 * or NULL (zeros: a sequence start); state_out: [b, Cc, W - 1] or NULL, the
 * last W - 1 inputs (state_in's entries when L < W - 1), so that a sequence
 * cut in two and run with state_out -> state_in gives the same u. */
int orc_conv1d(int64_t batch, int64_t seqlen, int64_t channels, int64_t width,
               const double *x, const double *w, const double *bias,
               const double *state_in, int act, double *u, double *state_out);

/* The Mamba-2 mixer's gated RMS norm over each row of `width` values (a
 * token's whole mixer width, heads x head_dim): g = y * silu(z) (g = y when
 * z is NULL), out = g / sqrt(mean(g^2) + eps) * weight (weight NULL = 1).
 * y, z, out: [rows, width]; weight: [width]. */
int orc_gated_rmsnorm(int64_t rows, int64_t width, double eps, const double *y,
                      const double *z, const double *weight, double *out);

/* The hidden attention of the Mamba-2 (SSD) map ("Mamba-2", nnterp
 * encyclopedia, "The hidden attention"): per head, the causal [seq, seq]
 * matrix with y_t = sum_s alpha[t, s] x_s + D x_t (zero initial state),
 *   alpha[t, s] = (C_t . B_s) * exp(decays_{s+1} + ... + decays_t) * betas_s
 * for s <= t and 0 above the diagonal, with betas = softplus(dt + dt_bias)
 * (when ORC_SOFTPLUS) and decays = betas * A_h.  dt: [b, L, H]; B, Cm:
 * [b, L, G, N]; A, dt_bias: [H]; alpha: [b, H, L, L] (query t, key s). */
int orc_m2_attention(int64_t batch, int64_t seqlen, int64_t heads, int64_t state,
                     int64_t groups, uint32_t flags, const double *dt, const double *B,
                     const double *Cm, const double *A, const double *dt_bias, double *alpha);

/* Elementwise helpers exposed for the pins. */
double orc_softplus(double v);
double orc_silu(double v);
/* Weightless RMS norm of rows of length n: out = v / sqrt(mean(v^2) + eps). */
void orc_rms_rows(int64_t rows, int64_t n, double eps, const double *in,
                  double *out);

#ifdef __cplusplus
}
#endif
#endif
