"""Coefficients of the FMA-pipe exp2 used by the Mamba-1 scan kernel.

Method: Cody-Waite range reduction x = j + f with j = round(x), f in
[-1/2, 1/2], then 2^f ~ p(f) = 1 + f (c1 + c2 f + ... + c5 f^4), i.e. the
constant term is exactly 1 so that 2^0 = 1 exactly (a zero step keeps the
state bit for bit).  The c_k are a weighted least-squares fit of
(2^f - 1) / f on Chebyshev nodes (weight 2^-f, so the error is relative),
which is close to the minimax polynomial.  2^j is applied by adding j to
the exponent field.

Running this prints the float32 coefficients and the maximum relative error
of the float32 Horner evaluation over a dense grid of f.
"""
import numpy as np

DEGREE = 5


def fit(degree=DEGREE, nodes=4000):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)           # Chebyshev nodes on [-1/2, 1/2]
    g = np.where(np.abs(f) < 1e-12, np.log(2.0), np.expm1(f * np.log(2.0)) / f)
    # relative error of 1 + f q(f) against 2^f is f (q - g) / 2^f
    w = np.abs(f) / np.exp2(f)
    V = np.vander(f, degree, increasing=True)              # columns f^0 .. f^(degree-1)
    coef, *_ = np.linalg.lstsq(V * w[:, None], g * w, rcond=None)
    return coef.astype(np.float32)                          # c1 .. c_degree


def eval_f32(coef, f):
    f = f.astype(np.float32)
    acc = np.float32(coef[-1])
    for c in coef[-2::-1]:
        acc = np.float32(acc * f + np.float32(c))
    return np.float32(np.float32(acc * f) + np.float32(1.0))


def max_rel_error(coef, n=2000001):
    f = np.linspace(-0.5, 0.5, n)
    p = eval_f32(coef, f).astype(np.float64)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, v in enumerate(c, 1):
        print("c%d = %.9e  (0x%08x)" % (i, v, np.float32(v).view(np.uint32)))
    print("max relative error of the float32 evaluation: %.3e" % max_rel_error(c))
