"""Fit of the polynomial that evaluates 2^f on the FMA pipe (for |f| <= 1/2).

The forward softmax computes one exp2 per score.  The special-function unit
that runs ex2.approx has a fraction of the FMA pipe's throughput, so the
kernel evaluates a share of the exponentials with plain fp32 arithmetic:

    x = n + f,  n = round(x),  |f| <= 1/2      (range reduction)
    2^x = 2^n * p(f),  p(f) ~ 2^f              (polynomial on the FMA pipe)

with 2^n applied by adding n to the exponent field of p(f).  This script
derives p: the degree-3 polynomial minimising the maximum RELATIVE error
|p(f) / 2^f - 1| on [-1/2, 1/2], found as a linear programme over a dense grid
(the discrete minimax / Chebyshev approximation problem), then checks the
error of the fp32 evaluation order the kernel uses.  Its output is the set of
constants in fwd_kernel.cuh and the bound the tests use.

    python exp2_poly_fit.py
"""
from __future__ import annotations

import numpy as np
from scipy.optimize import linprog

DEGREE = 3


def fit(degree: int = DEGREE, n_grid: int = 4001):
    f = np.linspace(-0.5, 0.5, n_grid)
    y = np.exp2(f)
    # variables: c_0..c_degree, t ; minimise t subject to |sum c_k f^k - y| <= t*y
    V = np.vander(f, degree + 1, increasing=True)
    ones = y[:, None]
    A = np.vstack([np.hstack([V, -ones]), np.hstack([-V, -ones])])
    b = np.concatenate([y, -y])
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1) + [(0, None)],
                  method="highs")
    assert res.success, res.message
    return res.x[:-1], res.x[-1]


def eval_fp32(coeffs, f):
    """Horner in fp32, the order the kernel uses: ((c3 f + c2) f + c1) f + c0."""
    c = [np.float32(v) for v in coeffs]
    f = np.asarray(f, np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    coeffs, err = fit()
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.max(np.abs(eval_fp32(coeffs, f).astype(np.float64) / np.exp2(f) - 1.0))
    for k, c in enumerate(coeffs):
        print(f"c{k} = {np.float32(c)!r}f   ({c:.17g})")
    print(f"minimax relative error {err:.3e}; fp32 Horner evaluation {rel:.3e}")
