/*
 * ssm_oracle.c -- float64 CPU oracle for the selective state-space scan.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product path.  It is a plain
 * token loop in the pages' order and notation; it does not chunk, block or
 * reorder the recurrence.  See ssm_oracle.h for the layouts and sources.
 *
 * Readings taken where the pages leave a step open:
 *   - softplus is evaluated exactly as max(v,0) + log1p(exp(-|v|)); no
 *     threshold, no clamp of the step ("Mamba-2", "A zero step skips a token
 *     exactly": time_step_limit (0, inf), nothing is clamped).
 *   - token t's own decay multiplies h_{t-1}; y_t reads h_t after token t's
 *     write, in the scan and the decode step alike ("Mamba", "The state" and
 *     the read-order warning; "Mamba", tokentrails, "Code").
 *   - the silu(z) gate multiplies the whole y = C.h + D*x ("Falcon-Mamba",
 *     "The block, in order": out_proj(y * silu(z)) with y including D*u).
 *   - the Falcon norm on the step acts on dt_raw's last axis (the channels),
 *     then dt_bias is added, then softplus; B and C are normed over N.
 */
#include "ssm_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

double orc_softplus(double v) { return fmax(v, 0.0) + log1p(exp(-fabs(v))); }

/* silu(z) = z * sigmoid(z) = z / (1 + exp(-z)). */
double orc_silu(double v) { return v / (1.0 + exp(-v)); }

/* Weightless RMS norm ("Falcon-Mamba", "Where the norms sit"): each row of
 * n values is divided by sqrt(mean(v^2) + eps); there is no gain. */
void orc_rms_rows(int64_t rows, int64_t n, double eps, const double *in,
                  double *out) {
  for (int64_t r = 0; r < rows; ++r) {
    const double *v = in + r * n;
    double ss = 0.0;
    for (int64_t i = 0; i < n; ++i) ss += v[i] * v[i];
    double inv = 1.0 / sqrt(ss / (double)n + eps);
    for (int64_t i = 0; i < n; ++i) out[r * n + i] = v[i] * inv;
  }
}

/* ---------------------------------------------------------------- threads */

typedef void (*unit_fn)(void *ctx, int64_t unit);
typedef struct {
  unit_fn fn;
  void *ctx;
  int64_t begin, end;
} span_t;

static void *run_span(void *p) {
  span_t *s = (span_t *)p;
  for (int64_t u = s->begin; u < s->end; ++u) s->fn(s->ctx, u);
  return NULL;
}

/* Runs fn(ctx, u) for u in [0, units), split into contiguous spans. */
static int for_units(int64_t units, int nthreads, unit_fn fn, void *ctx) {
  if (nthreads < 1) nthreads = 1;
  if ((int64_t)nthreads > units) nthreads = (int)(units > 0 ? units : 1);
  if (nthreads == 1) {
    span_t s = {fn, ctx, 0, units};
    run_span(&s);
    return 0;
  }
  pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  span_t *sp = (span_t *)malloc(sizeof(span_t) * (size_t)nthreads);
  if (!tid || !sp) {
    free(tid);
    free(sp);
    return -1;
  }
  for (int i = 0; i < nthreads; ++i) {
    sp[i].fn = fn;
    sp[i].ctx = ctx;
    sp[i].begin = units * i / nthreads;
    sp[i].end = units * (i + 1) / nthreads;
    pthread_create(&tid[i], NULL, run_span, &sp[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(tid[i], NULL);
  free(tid);
  free(sp);
  return 0;
}

/* ------------------------------------------------------------- Mamba-1 */

typedef struct {
  int64_t Bt, L, Cn, N, G;
  uint32_t flags;
  const double *x, *dt, *z, *B, *Cm, *A, *D, *dt_bias, *h0;
  const double *dt_scale; /* [b, L] RMS factor of dt_raw, or NULL */
  const double *bc_norm;  /* [b, L, G, 2, N]: normed B then C, or NULL */
  double *y, *h_last, *states;
  int64_t t_write;            /* token whose state is replaced, or -1       */
  const double *state_write;  /* [b, C, N]: the state written at t_write     */
} m1_ctx;

/* One (batch, channel) pair: the token loop of the recurrence
 *   h = exp(dt * A[c, :]) * h + dt * B_t * x_t,   y_t = C_t . h + D[c] x_t
 * ("Mamba", nnterp guide, intro; tokentrails "Code"). */
static void m1_unit(void *p, int64_t u) {
  const m1_ctx *k = (const m1_ctx *)p;
  const int64_t b = u / k->Cn, c = u % k->Cn;
  const int64_t L = k->L, Cn = k->Cn, N = k->N, G = k->G;
  const int64_t g = c / (Cn / G);
  double h[1024];
  for (int64_t n = 0; n < N; ++n)
    h[n] = k->h0 ? k->h0[(b * Cn + c) * N + n] : 0.0;
  const double Dc = k->D ? k->D[c] : 0.0;
  const double bias = k->dt_bias ? k->dt_bias[c] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    const int64_t i = (b * L + t) * Cn + c;
    double d = k->dt[i];
    if (k->dt_scale) d *= k->dt_scale[b * L + t];
    d += bias;
    if (k->flags & ORC_SOFTPLUS) d = orc_softplus(d);
    const double xv = k->x[i];
    const double *Bt, *Ct;
    if (k->bc_norm) {
      Bt = k->bc_norm + (((b * L + t) * G + g) * 2 + 0) * N;
      Ct = k->bc_norm + (((b * L + t) * G + g) * 2 + 1) * N;
    } else {
      Bt = k->B + ((b * L + t) * G + g) * N;
      Ct = k->Cm + ((b * L + t) * G + g) * N;
    }
    double acc = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      h[n] = exp(d * k->A[c * N + n]) * h[n] + d * Bt[n] * xv;
      acc += Ct[n] * h[n];
    }
    if (k->state_write && t == k->t_write) {
      /* A state written at token t replaces h_t: y_t reads the written
       * state, and later tokens continue from it ("Mamba", nnterp guide,
       * "The state": a write at token t changes token t's own output). */
      acc = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        h[n] = k->state_write[(b * Cn + c) * N + n];
        acc += Ct[n] * h[n];
      }
    }
    double yv = acc + Dc * xv;
    if (k->z) yv *= orc_silu(k->z[i]);
    k->y[i] = yv;
    if (k->states)
      memcpy(k->states + ((b * L + t) * Cn + c) * N, h, sizeof(double) * N);
  }
  if (k->h_last) memcpy(k->h_last + (b * Cn + c) * N, h, sizeof(double) * N);
}

static int m1_scan_impl(int64_t batch, int64_t seqlen, int64_t channels, int64_t state,
                        int64_t groups, uint32_t flags, double rms_eps,
                        const double *x, const double *dt, const double *z,
                        const double *B, const double *Cm, const double *A,
                        const double *D, const double *dt_bias, const double *h0,
                        double *y, double *h_last, double *states, int nthreads,
                        int64_t t_write, const double *state_write) {
  if (state > 1024 || groups < 1 || channels % groups) return -1;
  m1_ctx k = {batch, seqlen, channels, state, groups, flags, x, dt, z, B, Cm,
              A, D, dt_bias, h0, NULL, NULL, y, h_last, states, t_write, state_write};
  double *dt_scale = NULL, *bc_norm = NULL;
  if (flags & ORC_RMS_DT) {
    /* One factor per (b, t): 1 / sqrt(mean over channels of dt_raw^2 + eps). */
    dt_scale = (double *)malloc(sizeof(double) * (size_t)(batch * seqlen));
    if (!dt_scale) return -2;
    for (int64_t r = 0; r < batch * seqlen; ++r) {
      double ss = 0.0;
      for (int64_t c = 0; c < channels; ++c)
        ss += dt[r * channels + c] * dt[r * channels + c];
      dt_scale[r] = 1.0 / sqrt(ss / (double)channels + rms_eps);
    }
    k.dt_scale = dt_scale;
  }
  if (flags & ORC_RMS_BC) {
    const int64_t rows = batch * seqlen * groups;
    bc_norm = (double *)malloc(sizeof(double) * (size_t)(rows * 2 * state));
    if (!bc_norm) {
      free(dt_scale);
      return -2;
    }
    for (int64_t r = 0; r < rows; ++r) {
      orc_rms_rows(1, state, rms_eps, B + r * state, bc_norm + (r * 2) * state);
      orc_rms_rows(1, state, rms_eps, Cm + r * state,
                   bc_norm + (r * 2 + 1) * state);
    }
    k.bc_norm = bc_norm;
  }
  int rc = for_units(batch * channels, nthreads, m1_unit, &k);
  free(dt_scale);
  free(bc_norm);
  return rc;
}

int orc_m1_scan(int64_t batch, int64_t seqlen, int64_t channels, int64_t state,
                int64_t groups, uint32_t flags, double rms_eps,
                const double *x, const double *dt, const double *z,
                const double *B, const double *Cm, const double *A,
                const double *D, const double *dt_bias, const double *h0,
                double *y, double *h_last, double *states, int nthreads) {
  return m1_scan_impl(batch, seqlen, channels, state, groups, flags, rms_eps, x, dt, z, B, Cm,
                      A, D, dt_bias, h0, y, h_last, states, nthreads, -1, NULL);
}

int orc_m1_scan_write(int64_t batch, int64_t seqlen, int64_t channels, int64_t state,
                      int64_t groups, uint32_t flags, double rms_eps,
                      const double *x, const double *dt, const double *z,
                      const double *B, const double *Cm, const double *A,
                      const double *D, const double *dt_bias, const double *h0,
                      int64_t t_write, const double *state_write,
                      double *y, double *h_last, double *states, int nthreads) {
  if (t_write < 0 || t_write >= seqlen || !state_write) return -1;
  return m1_scan_impl(batch, seqlen, channels, state, groups, flags, rms_eps, x, dt, z, B, Cm,
                      A, D, dt_bias, h0, y, h_last, states, nthreads, t_write, state_write);
}

/* ------------------------------------------------------------- Mamba-2 */

typedef struct {
  int64_t Bt, L, H, P, N, G;
  uint32_t flags;
  const double *x, *dt, *z, *B, *Cm, *A, *D, *dt_bias, *h0;
  double *y, *h_last, *states;
} m2_ctx;

/* One (batch, head) pair.  The head keeps an N x P state (key side first);
 * each token decays it by one scalar exp(dt A_h) and adds the outer product
 * dt * B_t x_t^T; y_t = C_t^T h_t + D_h x_t
 * ("Mamba-2", "The mixer's values" and "The state"). */
static void m2_unit(void *p, int64_t u) {
  const m2_ctx *k = (const m2_ctx *)p;
  const int64_t b = u / k->H, hd = u % k->H;
  const int64_t L = k->L, H = k->H, P = k->P, N = k->N, G = k->G;
  const int64_t g = hd / (H / G);
  double *S = (double *)malloc(sizeof(double) * (size_t)(N * P));
  if (!S) return;
  for (int64_t e = 0; e < N * P; ++e)
    S[e] = k->h0 ? k->h0[(b * H + hd) * N * P + e] : 0.0;
  const double Dh = k->D ? k->D[hd] : 0.0;
  const double bias = k->dt_bias ? k->dt_bias[hd] : 0.0;
  const double Ah = k->A[hd];
  for (int64_t t = 0; t < L; ++t) {
    double d = k->dt[(b * L + t) * H + hd] + bias;
    if (k->flags & ORC_SOFTPLUS) d = orc_softplus(d);
    const double a = exp(d * Ah);
    const double *Bt = k->B + ((b * L + t) * G + g) * N;
    const double *Ct = k->Cm + ((b * L + t) * G + g) * N;
    const double *xt = k->x + ((b * L + t) * H + hd) * P;
    for (int64_t n = 0; n < N; ++n)
      for (int64_t q = 0; q < P; ++q)
        S[n * P + q] = a * S[n * P + q] + d * Bt[n] * xt[q];
    for (int64_t q = 0; q < P; ++q) {
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) acc += Ct[n] * S[n * P + q];
      double yv = acc + Dh * xt[q];
      if (k->z) yv *= orc_silu(k->z[((b * L + t) * H + hd) * P + q]);
      k->y[((b * L + t) * H + hd) * P + q] = yv;
    }
    if (k->states)
      memcpy(k->states + ((b * L + t) * H + hd) * N * P, S,
             sizeof(double) * (size_t)(N * P));
  }
  if (k->h_last)
    memcpy(k->h_last + (b * H + hd) * N * P, S, sizeof(double) * (size_t)(N * P));
  free(S);
}

int orc_m2_scan(int64_t batch, int64_t seqlen, int64_t heads, int64_t head_dim,
                int64_t state, int64_t groups, uint32_t flags,
                const double *x, const double *dt, const double *z,
                const double *B, const double *Cm, const double *A,
                const double *D, const double *dt_bias, const double *h0,
                double *y, double *h_last, double *states, int nthreads) {
  if (groups < 1 || heads % groups) return -1;
  m2_ctx k = {batch, seqlen, heads, head_dim, state, groups, flags, x, dt, z,
              B, Cm, A, D, dt_bias, h0, y, h_last, states};
  return for_units(batch * heads, nthreads, m2_unit, &k);
}

/* ---------------------------------------------------------- decode step */

/* One new token against a cached state.  The state is updated first and
 * y is read from the updated state ("Mamba", nnterp guide, "The state" and
 * "Read order on a decode step"). */
int orc_m1_step(int64_t batch, int64_t channels, int64_t state, int64_t groups,
                uint32_t flags, double rms_eps,
                const double *x, const double *dt, const double *z,
                const double *B, const double *Cm, const double *A,
                const double *D, const double *dt_bias,
                double *state_io, double *y) {
  if (groups < 1 || channels % groups || state > 1024) return -1;
  for (int64_t b = 0; b < batch; ++b) {
    double dscale = 1.0;
    if (flags & ORC_RMS_DT) {
      double ss = 0.0;
      for (int64_t c = 0; c < channels; ++c)
        ss += dt[b * channels + c] * dt[b * channels + c];
      dscale = 1.0 / sqrt(ss / (double)channels + rms_eps);
    }
    for (int64_t c = 0; c < channels; ++c) {
      const int64_t g = c / (channels / groups);
      double Bn[1024], Cn[1024];
      if (flags & ORC_RMS_BC) {
        orc_rms_rows(1, state, rms_eps, B + (b * groups + g) * state, Bn);
        orc_rms_rows(1, state, rms_eps, Cm + (b * groups + g) * state, Cn);
      } else {
        memcpy(Bn, B + (b * groups + g) * state, sizeof(double) * state);
        memcpy(Cn, Cm + (b * groups + g) * state, sizeof(double) * state);
      }
      double d = dt[b * channels + c];
      if (flags & ORC_RMS_DT) d *= dscale;
      d += dt_bias ? dt_bias[c] : 0.0;
      if (flags & ORC_SOFTPLUS) d = orc_softplus(d);
      const double xv = x[b * channels + c];
      double *h = state_io + (b * channels + c) * state;
      /* update ... */
      for (int64_t n = 0; n < state; ++n)
        h[n] = exp(d * A[c * state + n]) * h[n] + d * Bn[n] * xv;
      /* ... then read */
      double acc = 0.0;
      for (int64_t n = 0; n < state; ++n) acc += Cn[n] * h[n];
      double yv = acc + (D ? D[c] : 0.0) * xv;
      if (z) yv *= orc_silu(z[b * channels + c]);
      y[b * channels + c] = yv;
    }
  }
  return 0;
}

int orc_m2_step(int64_t batch, int64_t heads, int64_t head_dim, int64_t state,
                int64_t groups, uint32_t flags,
                const double *x, const double *dt, const double *z,
                const double *B, const double *Cm, const double *A,
                const double *D, const double *dt_bias,
                double *state_io, double *y) {
  if (groups < 1 || heads % groups) return -1;
  const int64_t P = head_dim, N = state;
  for (int64_t b = 0; b < batch; ++b) {
    for (int64_t hd = 0; hd < heads; ++hd) {
      const int64_t g = hd / (heads / groups);
      double d = dt[b * heads + hd] + (dt_bias ? dt_bias[hd] : 0.0);
      if (flags & ORC_SOFTPLUS) d = orc_softplus(d);
      const double a = exp(d * A[hd]);
      const double *Bg = B + (b * groups + g) * N;
      const double *Cg = Cm + (b * groups + g) * N;
      const double *xh = x + (b * heads + hd) * P;
      double *S = state_io + (b * heads + hd) * N * P;
      for (int64_t n = 0; n < N; ++n)
        for (int64_t q = 0; q < P; ++q)
          S[n * P + q] = a * S[n * P + q] + d * Bg[n] * xh[q];
      for (int64_t q = 0; q < P; ++q) {
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) acc += Cg[n] * S[n * P + q];
        double yv = acc + (D ? D[hd] : 0.0) * xh[q];
        if (z) yv *= orc_silu(z[(b * heads + hd) * P + q]);
        y[(b * heads + hd) * P + q] = yv;
      }
    }
  }
  return 0;
}

/* ------------------------------------------------ quadratic (brute force) */

/* "Mamba-2", "The hidden attention": per head the scan is the causal map
 *   y_t = sum_{s<=t} alpha[t, s] x_s + D x_t,
 *   alpha[t, s] = (C_t . B_s) * exp(decays_{s+1} + ... + decays_t) * betas_s,
 * with decays = betas * A.  The sum of decays is formed term by term (no
 * cumulative-sum difference), and a non-zero initial state enters through
 * C_t . exp(decays_1 + ... + decays_t) h0. */
int orc_m2_quadratic(int64_t batch, int64_t seqlen, int64_t heads,
                     int64_t head_dim, int64_t state, int64_t groups,
                     const double *x, const double *betas, const double *z,
                     const double *B, const double *Cm, const double *A,
                     const double *D, const double *h0, double *y) {
  if (groups < 1 || heads % groups) return -1;
  const int64_t L = seqlen, H = heads, P = head_dim, N = state, G = groups;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t hd = 0; hd < H; ++hd) {
      const int64_t g = hd / (H / G);
      for (int64_t t = 0; t < L; ++t) {
        const double *Ct = Cm + ((b * L + t) * G + g) * N;
        for (int64_t q = 0; q < P; ++q) {
          double acc = 0.0;
          for (int64_t s = 0; s <= t; ++s) {
            const double *Bs = B + ((b * L + s) * G + g) * N;
            double cb = 0.0;
            for (int64_t n = 0; n < N; ++n) cb += Ct[n] * Bs[n];
            double dsum = 0.0;
            for (int64_t r = s + 1; r <= t; ++r)
              dsum += betas[(b * L + r) * H + hd] * A[hd];
            acc += cb * exp(dsum) * betas[(b * L + s) * H + hd] *
                   x[((b * L + s) * H + hd) * P + q];
          }
          if (h0) {
            double dsum = 0.0;
            for (int64_t r = 0; r <= t; ++r)
              dsum += betas[(b * L + r) * H + hd] * A[hd];
            double ch = 0.0;
            for (int64_t n = 0; n < N; ++n)
              ch += Ct[n] * h0[((b * H + hd) * N + n) * P + q];
            acc += exp(dsum) * ch;
          }
          const int64_t i = ((b * L + t) * H + hd) * P + q;
          double yv = acc + (D ? D[hd] : 0.0) * x[i];
          if (z) yv *= orc_silu(z[i]);
          y[i] = yv;
        }
      }
    }
  return 0;
}

/* The Mamba-1 counterpart: A is per channel and state index, so the decay
 * factor is exp(sum_{r=s+1..t} betas_r A[c, n]) inside the sum over n
 * ("Mamba", nnterp guide, "The values": decays has a state axis). */
int orc_m1_quadratic(int64_t batch, int64_t seqlen, int64_t channels,
                     int64_t state, int64_t groups,
                     const double *x, const double *betas, const double *z,
                     const double *B, const double *Cm, const double *A,
                     const double *D, const double *h0, double *y) {
  if (groups < 1 || channels % groups) return -1;
  const int64_t L = seqlen, Cn = channels, N = state, G = groups;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t c = 0; c < Cn; ++c) {
      const int64_t g = c / (Cn / G);
      for (int64_t t = 0; t < L; ++t) {
        const double *Ct = Cm + ((b * L + t) * G + g) * N;
        double acc = 0.0;
        for (int64_t s = 0; s <= t; ++s) {
          const double *Bs = B + ((b * L + s) * G + g) * N;
          for (int64_t n = 0; n < N; ++n) {
            double dsum = 0.0;
            for (int64_t r = s + 1; r <= t; ++r)
              dsum += betas[(b * L + r) * Cn + c] * A[c * N + n];
            acc += Ct[n] * Bs[n] * exp(dsum) * betas[(b * L + s) * Cn + c] *
                   x[(b * L + s) * Cn + c];
          }
        }
        if (h0)
          for (int64_t n = 0; n < N; ++n) {
            double dsum = 0.0;
            for (int64_t r = 0; r <= t; ++r)
              dsum += betas[(b * L + r) * Cn + c] * A[c * N + n];
            acc += Ct[n] * exp(dsum) * h0[(b * Cn + c) * N + n];
          }
        const int64_t i = (b * L + t) * Cn + c;
        double yv = acc + (D ? D[c] : 0.0) * x[i];
        if (z) yv *= orc_silu(z[i]);
        y[i] = yv;
      }
    }
  return 0;
}

/* Causal depthwise convolution ("Mamba-2", module tree and "The mixer's
 * values"; "Mamba", tokentrails, "Code"): the module's Conv1d with padding
 * W - 1 on both ends and the output cut to the first L positions is, per
 * channel, a weighted sum of the current input and the W - 1 before it,
 * weight k multiplying the input W - 1 - k tokens back; inputs before the
 * sequence start come from state_in (zero without one). */
static double conv_in(const double *x, const double *state_in, int64_t b, int64_t L, int64_t Cc,
                      int64_t W, int64_t c, int64_t tau) {
  if (tau >= 0) return x[(b * L + tau) * Cc + c];
  if (!state_in) return 0.0;
  return state_in[(b * Cc + c) * (W - 1) + (W - 1) + tau];
}

int orc_conv1d(int64_t batch, int64_t seqlen, int64_t channels, int64_t width,
               const double *x, const double *w, const double *bias,
               const double *state_in, int act, double *u, double *state_out) {
  const int64_t L = seqlen, Cc = channels, W = width;
  if (batch < 0 || L < 0 || Cc <= 0 || W <= 0 || !w) return 1;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t c = 0; c < Cc; ++c) {
      for (int64_t t = 0; t < L; ++t) {
        double acc = bias ? bias[c] : 0.0;
        for (int64_t k = 0; k < W; ++k)
          acc += w[c * W + k] * conv_in(x, state_in, b, L, Cc, W, c, t - (W - 1) + k);
        u[(b * L + t) * Cc + c] = act ? orc_silu(acc) : acc;
      }
      if (state_out)
        for (int64_t j = 0; j < W - 1; ++j)
          state_out[(b * Cc + c) * (W - 1) + j] =
              conv_in(x, state_in, b, L, Cc, W, c, L - (W - 1) + j);
    }
  return 0;
}

/* Gated RMS norm ("Mamba-2", "The mixer's values" and the paragraph on the
 * block's norms): the gate first, y * silu(z), then one RMS norm over the
 * whole row -- the mixer's full width, not per group -- then the weight. */
int orc_gated_rmsnorm(int64_t rows, int64_t width, double eps, const double *y,
                      const double *z, const double *weight, double *out) {
  if (rows < 0 || width <= 0 || !y || !out) return 1;
  for (int64_t r = 0; r < rows; ++r) {
    const double *yr = y + r * width;
    double *o = out + r * width;
    double ss = 0.0;
    for (int64_t i = 0; i < width; ++i) {
      const double g = z ? yr[i] * orc_silu(z[r * width + i]) : yr[i];
      o[i] = g;
      ss += g * g;
    }
    const double inv = 1.0 / sqrt(ss / (double)width + eps);
    for (int64_t i = 0; i < width; ++i) o[i] = o[i] * inv * (weight ? weight[i] : 1.0);
  }
  return 0;
}

/* The hidden attention ("Mamba-2", "The hidden attention"), by its
 * definition: the decay between key s and query t is the sum of the decays
 * of tokens s+1 .. t, summed term by term. */
int orc_m2_attention(int64_t batch, int64_t seqlen, int64_t heads, int64_t state,
                     int64_t groups, uint32_t flags, const double *dt, const double *B,
                     const double *Cm, const double *A, const double *dt_bias, double *alpha) {
  const int64_t L = seqlen, H = heads, N = state, G = groups;
  if (batch < 0 || L < 0 || H <= 0 || N <= 0 || G <= 0 || H % G || !alpha) return 1;
  double *beta = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  if (!beta) return 2;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t h = 0; h < H; ++h) {
      const int64_t g = h / (H / G);
      for (int64_t t = 0; t < L; ++t) {
        double d = dt[(b * L + t) * H + h] + (dt_bias ? dt_bias[h] : 0.0);
        if (flags & ORC_SOFTPLUS) d = orc_softplus(d);
        beta[t] = d;
      }
      for (int64_t t = 0; t < L; ++t)
        for (int64_t s2 = 0; s2 < L; ++s2) {
          double v = 0.0;
          if (s2 <= t) {
            double cb = 0.0;
            for (int64_t n = 0; n < N; ++n)
              cb += Cm[((b * L + t) * G + g) * N + n] * B[((b * L + s2) * G + g) * N + n];
            double dsum = 0.0;
            for (int64_t r = s2 + 1; r <= t; ++r) dsum += beta[r] * A[h];
            v = cb * exp(dsum) * beta[s2];
          }
          alpha[((b * H + h) * L + t) * L + s2] = v;
        }
    }
  free(beta);
  return 0;
}
