"""Coefficients of the cubic the softmax kernels use for part of their base-2
exponentials (the rest go to the MUFU ex2 unit).

2^x is split as 2^j * 2^f with j = rint(x) and f = x - j in [-0.5, 0.5]
(Cody and Waite's argument reduction, trivial in base 2: 2^j is built
directly as an exponent field).  2^f is approximated by a cubic whose
coefficients minimise the maximum RELATIVE error on [-0.5, 0.5]; the fit
below is an iteratively reweighted least-squares approximation of that
minimax problem on Chebyshev nodes.  The kernels round the result to bf16
(relative half-ulp 2^-9 = 1.95e-3), so the cubic's 7.5e-5 is far inside the
output's own rounding.  `python exp2_fit.py` prints the coefficients as the
C initialisers used in csrc/sm100.cuh; tests/test_exp2_poly.py checks that
the header matches this fit and emulates the kernel's fp32 steps.
"""
import numpy as np


def fit(deg=3, nodes=4001, iters=60):
    f = np.cos(np.linspace(0.0, np.pi, nodes)) * 0.5
    target = 2.0 ** f
    A = np.vstack([f ** k for k in range(deg + 1)]).T / target[:, None]
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(A * w[:, None], w, rcond=None)
        err = A @ c - 1.0
        w = w * (1.0 + 50.0 * np.abs(err) / np.abs(err).max())
        w /= w.mean()
    return c


def max_rel_error(c, n=200001):
    x = np.linspace(-0.5, 0.5, n)
    return float(np.abs(np.polyval(c[::-1], x) / 2.0 ** x - 1.0).max())


if __name__ == "__main__":
    c = fit()
    print("max relative error %.3e" % max_rel_error(c))
    for k, v in enumerate(c):
        print("c%d = %.9ef" % (k, np.float32(v)))
