"""Fit of the odd polynomial that evaluates tanh(y) on the FMA pipe (|y| <= 1/2).

With a softcap c every scaled score s becomes c tanh(s / c) before the
softmax.  Taking tanh through the special-function unit (one ex2 and one
reciprocal, on top of the softmax's own ex2) triples that unit's work per
score, and it is already the forward's limit.  For |y| <= Y0 the forward
instead evaluates

    tanh(y) = y * P(y^2),   P(u) = a0 + a1 u + ... + a4 u^4

with fp32 fused multiply-adds; a block whose scores all satisfy
|s scale / c| <= Y0 takes this path, any other block the exact identity
tanh(y) = 1 - 2 / (e^{2y} + 1).  P is the degree-4 polynomial minimising the
maximum RELATIVE error |P(y^2) / (tanh(y) / y) - 1| on [0, Y0], found as a
linear programme over a dense grid (the discrete minimax problem) in the
Chebyshev basis of u (which keeps the programme well conditioned), then
converted to monomials.  The script prints the constants used in ptx.cuh and
the error of the fp32 evaluation order the kernel uses.

    python tanh_poly_fit.py
"""
from __future__ import annotations

import numpy as np
from numpy.polynomial import chebyshev as C
from scipy.optimize import linprog

Y0 = 0.5
DEGREE = 4


def fit(y0: float = Y0, degree: int = DEGREE, n_grid: int = 8001):
    y = np.linspace(1e-4, y0, n_grid)
    u = y * y
    g = np.tanh(y) / y
    umax = y0 * y0
    x = 2.0 * u / umax - 1.0  # u mapped to [-1, 1]
    V = C.chebvander(x, degree)
    # minimise t subject to |V c - g| <= t g
    A = np.vstack([np.hstack([V, -g[:, None]]), np.hstack([-V, -g[:, None]])])
    b = np.concatenate([g, -g])
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1) + [(0, None)],
                  method="highs", options={"primal_feasibility_tolerance": 1e-10,
                                           "dual_feasibility_tolerance": 1e-10})
    assert res.success, res.message
    cheb = res.x[:-1]
    # Chebyshev series in x = 2u/umax - 1 -> monomials in u
    mono_x = C.cheb2poly(cheb)
    mono_u = np.zeros(degree + 1)
    for k, ck in enumerate(mono_x):  # (2u/umax - 1)^k
        term = np.polynomial.polynomial.polypow([-1.0, 2.0 / umax], k)
        mono_u[: len(term)] += ck * term
    return mono_u


def eval_fp32(coeffs, y):
    """The kernel's order: u = y*y, Horner in u, then y * P, all in fp32."""
    a = [np.float32(v) for v in coeffs]
    y = np.asarray(y, np.float32)
    u = (y * y).astype(np.float32)
    p = a[-1]
    for k in range(len(a) - 2, -1, -1):
        p = (p * u + a[k]).astype(np.float32)
    return (y * p).astype(np.float32)


if __name__ == "__main__":
    coeffs = fit()
    y = np.linspace(-Y0, Y0, 400001)
    y = y[y != 0]
    exact = np.tanh(y.astype(np.float32).astype(np.float64))
    rel = np.max(np.abs(eval_fp32(coeffs, y).astype(np.float64) / exact - 1.0))
    for k, c in enumerate(coeffs):
        print(f"a{k} = {np.format_float_positional(np.float32(c))}f   ({c:.17g})")
    print(f"fp32 evaluation, max relative error on 0 < |y| <= {Y0}: {rel:.3e}")
