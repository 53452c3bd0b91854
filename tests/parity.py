"""Tolerances and comparison helpers for the GPU-vs-oracle parity tests.

Tolerance (normwise max-abs error): the largest absolute difference over a
tensor must not exceed ``rel * max|reference|``, with rel = 1e-4 for float32
I/O and 2e-2 for bfloat16 I/O, float32 state and arithmetic in both cases.
An elementwise relative bound would fail near zeros of y, which the scan
produces wherever C.h and D*x cancel."""
import numpy as np
import torch

REL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def to_np(t):
    return t.detach().float().cpu().double().numpy() if isinstance(t, torch.Tensor) else t


def assert_close_normwise(got, ref, rel, what=""):
    got, ref = to_np(got), np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), "%s: non-finite values" % what
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert err <= rel * scale + 1e-30, "%s: max|err| %.3e > %.1e * max|ref| (%.3e)" % (
        what, err, rel, scale)
    return err / scale if scale else 0.0
