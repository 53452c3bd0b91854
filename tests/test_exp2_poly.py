"""Accuracy of the FMA-pipe exp2 the Mamba-1 kernel uses for part of its
decays, checked on the CPU by evaluating the same float32 operations the
kernel performs (Cody-Waite reduction with the 1.5*2^23 + 127 rounding
constant, degree-5 polynomial, exponent-field scaling) against float64 2^x."""
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "..", "selective_state_space_28_b200", "csrc", "common.cuh")


def _coefficients():
    text = open(SRC).read()
    c = {int(k): np.float32(float(v)) for k, v in re.findall(r"kP(\d) = ([0-9.e+-]+)f", text)}
    magic = np.float32(float(re.search(r"kMagic = ([0-9.]+)f", text).group(1)))
    return [c[i] for i in range(1, 6)], magic


def _exp2_fma(d, A2, lim, coef, magic):
    """float32 emulation of one lane of exp2_fma2(d, A2, lim): 2^(d*A2) for
    d >= 0, A2 < 0."""
    f32 = np.float32
    d, A2, lim = f32(d), f32(A2), f32(lim)
    dc = np.minimum(d, lim)
    t = (dc.astype(np.float64) * A2 + magic).astype(f32)          # fmaf: one rounding
    r = f32(t - magic)
    f = (dc.astype(np.float64) * A2 - r).astype(f32)              # fmaf
    p = f32(coef[4])
    for c in (coef[3], coef[2], coef[1], coef[0]):
        p = (p.astype(np.float64) * f + c).astype(f32)
    p = (p.astype(np.float64) * f + 1.0).astype(f32)
    s = ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF).astype(np.uint32).view(f32)
    return (p * s).astype(f32)


def test_exp2_fma_accuracy_over_decay_range():
    coef, magic = _coefficients()
    rng = np.random.default_rng(0)
    d = rng.uniform(0, 2.0, 200000).astype(np.float32)
    A2 = -np.exp(rng.uniform(np.log(1e-3), np.log(60.0), d.size)).astype(np.float32)
    lim = (np.float32(-127.0) / A2).astype(np.float32)
    got = _exp2_fma(d, A2, lim, coef, magic).astype(np.float64)
    x = d.astype(np.float64) * A2.astype(np.float64)
    ref = np.exp2(x)
    normal = x > -125.0
    rel = np.abs(got[normal] / ref[normal] - 1.0)
    # polynomial error 1.9e-7 plus the float32 rounding of x = d*A2 (|x| * 2^-24 ln 2)
    bound = 2.5e-7 + np.abs(x[normal]) * 2.0 ** -24 * np.log(2.0) * 1.5
    assert np.all(rel <= bound), float(np.max(rel - bound))
    # far below the float32 range the decay is exactly zero, never garbage
    assert np.all(got[x < -127.0] == 0.0)


def test_exp2_fma_is_exact_at_zero_step():
    """d = 0 gives exactly 1, so a zero step keeps the state bit for bit."""
    coef, magic = _coefficients()
    A2 = -np.exp(np.linspace(-5, 5, 101)).astype(np.float32)
    got = _exp2_fma(np.zeros_like(A2), A2, np.float32(-127.0) / A2, coef, magic)
    assert np.all(got == np.float32(1.0))


def test_exp2_fma_matches_generator_fit():
    from importlib import util
    spec = util.spec_from_file_location(
        "gen", os.path.join(HERE, "..", "selective_state_space_28_b200", "csrc",
                            "gen_exp2_poly.py"))
    gen = util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    coef, _ = _coefficients()
    fit = gen.fit()
    assert np.allclose(np.array(coef), fit, rtol=1e-6, atol=0)
    assert gen.max_rel_error(fit, n=200001) < 2.0e-7
