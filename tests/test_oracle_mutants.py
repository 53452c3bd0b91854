"""Plant plausible mistakes in the oracle's C source and check that each one
fails at least one pin of tests/test_oracle_pins.py.

Each mutant is a one-place textual edit of oracle/ssm_oracle.c, compiled with
gcc into a temporary library and swapped in for the real one while the pins
run.  A mutant that passes every pin would mean the pins cannot see that
kind of mistake.
"""
import ctypes
import inspect
import os
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")

MUTANTS = {
    "drop_write_term": ("h[n] = exp(d * k->A[c * N + n]) * h[n] + d * Bt[n] * xv;",
                        "h[n] = exp(d * k->A[c * N + n]) * h[n];"),
    "decay_sign": ("h[n] = exp(d * k->A[c * N + n]) * h[n]",
                   "h[n] = exp(-d * k->A[c * N + n]) * h[n]"),
    "read_before_update": (
        "      h[n] = exp(d * k->A[c * N + n]) * h[n] + d * Bt[n] * xv;\n"
        "      acc += Ct[n] * h[n];",
        "      acc += Ct[n] * h[n];\n"
        "      h[n] = exp(d * k->A[c * N + n]) * h[n] + d * Bt[n] * xv;"),
    "drop_skip_term": ("double yv = acc + Dc * xv;", "double yv = acc;"),
    "gate_skips_D": ("    double yv = acc + Dc * xv;\n    if (k->z) yv *= orc_silu(k->z[i]);",
                     "    double yv = acc;\n    if (k->z) yv *= orc_silu(k->z[i]);\n"
                     "    yv += Dc * xv;"),
    "softplus_branch": ("log1p(exp(-fabs(v)))", "log1p(exp(-v))"),
    "group_index": ("const int64_t g = c / (Cn / G);\n  double h[1024];",
                    "const int64_t g = c % G;\n  double h[1024];"),
    "bias_after_softplus": (
        "    d += bias;\n    if (k->flags & ORC_SOFTPLUS) d = orc_softplus(d);\n    const double xv",
        "    if (k->flags & ORC_SOFTPLUS) d = orc_softplus(d);\n    d += bias;\n    const double xv"),
    "m2_reads_B_not_C": ("for (int64_t n = 0; n < N; ++n) acc += Ct[n] * S[n * P + q];\n      double yv = acc + Dh",
                         "for (int64_t n = 0; n < N; ++n) acc += Bt[n] * S[n * P + q];\n      double yv = acc + Dh"),
    "m2_decay_without_step": ("const double a = exp(d * Ah);", "const double a = exp(Ah);"),
    "m2_transposed_state": ("S[n * P + q] = a * S[n * P + q] + d * Bt[n] * xt[q];",
                            "S[n * P + q] = a * S[n * P + q] + d * Bt[q % N] * xt[n % P];"),
    "rms_dt_no_mean": ("dt_scale[r] = 1.0 / sqrt(ss / (double)channels + rms_eps);",
                       "dt_scale[r] = 1.0 / sqrt(ss + rms_eps);"),
    "rms_bc_swapped": ("orc_rms_rows(1, state, rms_eps, Cm + r * state,\n                   bc_norm + (r * 2 + 1) * state);",
                       "orc_rms_rows(1, state, rms_eps, B + r * state,\n                   bc_norm + (r * 2 + 1) * state);"),
    "quadratic_decay_off_by_one": ("for (int64_t r = s + 1; r <= t; ++r)\n              dsum += betas[(b * L + r) * H + hd] * A[hd];",
                                   "for (int64_t r = s; r <= t; ++r)\n              dsum += betas[(b * L + r) * H + hd] * A[hd];"),
    "h0_ignored": ("h[n] = k->h0 ? k->h0[(b * Cn + c) * N + n] : 0.0;", "h[n] = 0.0;"),
    "m2_step_read_before_update": (
        "      for (int64_t n = 0; n < N; ++n)\n        for (int64_t q = 0; q < P; ++q)\n"
        "          S[n * P + q] = a * S[n * P + q] + d * Bg[n] * xh[q];\n"
        "      for (int64_t q = 0; q < P; ++q) {\n        double acc = 0.0;\n"
        "        for (int64_t n = 0; n < N; ++n) acc += Cg[n] * S[n * P + q];\n"
        "        double yv = acc + (D ? D[hd] : 0.0) * xh[q];\n"
        "        if (z) yv *= orc_silu(z[(b * heads + hd) * P + q]);\n"
        "        y[(b * heads + hd) * P + q] = yv;\n      }",
        "      for (int64_t q = 0; q < P; ++q) {\n        double acc = 0.0;\n"
        "        for (int64_t n = 0; n < N; ++n) acc += Cg[n] * S[n * P + q];\n"
        "        double yv = acc + (D ? D[hd] : 0.0) * xh[q];\n"
        "        if (z) yv *= orc_silu(z[(b * heads + hd) * P + q]);\n"
        "        y[(b * heads + hd) * P + q] = yv;\n      }\n"
        "      for (int64_t n = 0; n < N; ++n)\n        for (int64_t q = 0; q < P; ++q)\n"
        "          S[n * P + q] = a * S[n * P + q] + d * Bg[n] * xh[q];"),
    "conv_weight_reversed": ("acc += w[c * W + k] * conv_in(x, state_in, b, L, Cc, W, c, t - (W - 1) + k);",
                             "acc += w[c * W + (W - 1 - k)] * conv_in(x, state_in, b, L, Cc, W, c, t - (W - 1) + k);"),
    "conv_not_causal": ("acc += w[c * W + k] * conv_in(x, state_in, b, L, Cc, W, c, t - (W - 1) + k);",
                        "acc += w[c * W + k] * conv_in(x, state_in, b, L, Cc, W, c, t - (W - 2) + k);"),
    "conv_state_newest_first": ("return state_in[(b * Cc + c) * (W - 1) + (W - 1) + tau];",
                                "return state_in[(b * Cc + c) * (W - 1) - 1 - tau];"),
    "conv_silu_before_bias": ("        double acc = bias ? bias[c] : 0.0;\n        for (int64_t k = 0; k < W; ++k)\n"
                              "          acc += w[c * W + k] * conv_in(x, state_in, b, L, Cc, W, c, t - (W - 1) + k);\n"
                              "        u[(b * L + t) * Cc + c] = act ? orc_silu(acc) : acc;",
                              "        double acc = 0.0;\n        for (int64_t k = 0; k < W; ++k)\n"
                              "          acc += w[c * W + k] * conv_in(x, state_in, b, L, Cc, W, c, t - (W - 1) + k);\n"
                              "        u[(b * L + t) * Cc + c] = (act ? orc_silu(acc) : acc) + (bias ? bias[c] : 0.0);"),
    "conv_state_out_off_by_one": ("conv_in(x, state_in, b, L, Cc, W, c, L - (W - 1) + j);",
                                  "conv_in(x, state_in, b, L, Cc, W, c, L - W + j);"),
    "gated_norm_gate_after": ("      const double g = z ? yr[i] * orc_silu(z[r * width + i]) : yr[i];\n      o[i] = g;\n      ss += g * g;",
                              "      const double g = yr[i];\n      o[i] = z ? g * orc_silu(z[r * width + i]) : g;\n      ss += g * g;"),
    "gated_norm_per_half": ("const double inv = 1.0 / sqrt(ss / (double)width + eps);\n    for (int64_t i = 0; i < width; ++i) o[i] = o[i] * inv * (weight ? weight[i] : 1.0);",
                            "double s1 = 0.0;\n    for (int64_t i = 0; i < width / 2; ++i) s1 += o[i] * o[i];\n"
                            "    for (int64_t i = 0; i < width; ++i) o[i] = o[i] * (1.0 / sqrt((i < width / 2 ? s1 : ss - s1) / (double)(width / 2) + eps)) * (weight ? weight[i] : 1.0);"),
    "gated_norm_no_weight": ("o[i] = o[i] * inv * (weight ? weight[i] : 1.0);", "o[i] = o[i] * inv;"),
    "gated_norm_eps_outside": ("const double inv = 1.0 / sqrt(ss / (double)width + eps);",
                               "const double inv = 1.0 / (sqrt(ss / (double)width) + eps);"),
    "state_write_keeps_old_readout": ("      acc = 0.0;\n      for (int64_t n = 0; n < N; ++n) {\n        h[n] = k->state_write[(b * Cn + c) * N + n];\n        acc += Ct[n] * h[n];\n      }",
                                      "      for (int64_t n = 0; n < N; ++n) {\n        h[n] = k->state_write[(b * Cn + c) * N + n];\n      }"),
    "state_write_one_token_late": ("if (k->state_write && t == k->t_write) {", "if (k->state_write && t == k->t_write + 1) {"),
    "attention_decay_includes_key": ("for (int64_t r = s2 + 1; r <= t; ++r) dsum += beta[r] * A[h];",
                                     "for (int64_t r = s2; r <= t; ++r) dsum += beta[r] * A[h];"),
    "attention_beta_of_query": ("v = cb * exp(dsum) * beta[s2];", "v = cb * exp(dsum) * beta[t];"),
    "attention_not_causal": ("if (s2 <= t) {", "if (1) {"),
}


def _pin_calls():
    """Every pin with every combination of its parametrize values (G as 1
    and 2 where it is a plain default)."""
    import itertools
    calls = []
    for name, fn in sorted(inspect.getmembers(pins, inspect.isfunction)):
        if not name.startswith("test_"):
            continue
        params = inspect.signature(fn).parameters
        axes = []
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            names = [n.strip() for n in mark.args[0].split(",")]
            vals = [v if len(names) > 1 else (v,) for v in mark.args[1]]
            axes.append([dict(zip(names, v)) for v in vals])
        if "G" in params and not any("G" in a[0] for a in axes if a):
            axes.append([{"G": 1}, {"G": 2}])
        for combo in itertools.product(*axes) if axes else [()]:
            kw = {}
            for d in combo:
                kw.update(d)
            calls.append((name, fn, kw))
    return calls


def _build_mutant(src, tmpdir, key):
    path = os.path.join(tmpdir, "mut_%s.c" % key)
    shutil_h = os.path.join(os.path.dirname(SRC), "ssm_oracle.h")
    with open(path, "w") as f:
        f.write(src.replace('#include "ssm_oracle.h"', '#include "%s"' % shutil_h))
    lib = os.path.join(tmpdir, "mut_%s.so" % key)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                    "-o", lib, path, "-lm", "-lpthread"], check=True)
    return lib


@pytest.mark.parametrize("key", sorted(MUTANTS))
def test_mutant_is_caught(key):
    with open(SRC) as f:
        src = f.read()
    old, new = MUTANTS[key]
    assert src.count(old) == 1, "mutation anchor for %s not unique/found" % key
    real = oracle._load()
    with tempfile.TemporaryDirectory() as tmp:
        mlib = ctypes.CDLL(_build_mutant(src.replace(old, new), tmp, key))
        for name in ("orc_m1_scan", "orc_m2_scan", "orc_m1_step", "orc_m2_step",
                     "orc_m2_quadratic", "orc_m1_quadratic", "orc_softplus", "orc_silu",
                     "orc_rms_rows", "orc_conv1d", "orc_gated_rmsnorm", "orc_m1_scan_write",
                     "orc_m2_attention"):
            getattr(mlib, name).argtypes = getattr(real, name).argtypes
            getattr(mlib, name).restype = getattr(real, name).restype
        caught = None
        oracle._lib = mlib
        try:
            for name, fn, kw in _pin_calls():
                try:
                    fn(**kw)
                except AssertionError:
                    caught = name
                    break
        finally:
            oracle._lib = real
    assert caught, "mutant %s passed every pin" % key
