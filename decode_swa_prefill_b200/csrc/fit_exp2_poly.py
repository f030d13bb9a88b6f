"""Fit of the polynomial the prefill kernel uses for part of its exp2 work.

Method: Cody-Waite style range reduction, 2^x = 2^j * 2^f with j = round(x)
and f = x - j in [-1/2, 1/2], and a polynomial p(f) ~ 2^f obtained by a
weighted least-squares fit on Chebyshev nodes of [-1/2, 1/2] (weights 2^-f,
so the fit minimises relative error; Chebyshev-node least squares is within a
small factor of the minimax polynomial).  The kernel applies 2^j by adding j
to the exponent field of p(f).

Run to print the coefficients (highest degree first) and the worst relative
error over a dense grid; the coefficients of exp2_poly2 in ptx.cuh were
produced by `python fit_exp2_poly.py 3`.
"""
import sys

import numpy as np


def fit(degree, nodes=64):
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))  # Chebyshev nodes in [-1/2, 1/2]
    target = np.exp2(f)
    V = np.vander(f, degree + 1)                         # columns f^degree ... f^0
    w = 1.0 / target                                     # relative error
    coef, *_ = np.linalg.lstsq(V * w[:, None], target * w, rcond=None)
    return coef


def max_rel_error(coef, n=200001):
    f = np.linspace(-0.5, 0.5, n)
    c32 = np.asarray(coef, dtype=np.float32)
    # evaluate in fp32 with Horner, as the kernel does
    p = np.full_like(f, c32[0], dtype=np.float32)
    f32 = f.astype(np.float32)
    for c in c32[1:]:
        p = (p * f32 + c).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = fit(deg)
    print("degree", deg)
    print("coefficients (f^%d .. f^0):" % deg, ", ".join("%.9ef" % x for x in c.astype(np.float32)))
    print("max relative error in fp32:", max_rel_error(c))
