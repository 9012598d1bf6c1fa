"""CPU check of the FMA-pipe softcap used by the forward softmax.

With a softcap c the forward turns each score s into c log2(e) tanh(s scale / c)
(the log2 domain of the softmax).  For blocks whose scores all have
|s scale / c| <= 1/2 it evaluates tanh as y P(y^2) with y = s scale / c and the
degree-4 polynomial of tanh_poly_fit.py, the constant c log2(e) folded into
P's coefficients.  Here the constants are read from ptx.cuh, the kernel's fp32
steps are replayed with numpy (round to nearest at every step, as the GPU
does), and the result is compared with the exact c log2(e) tanh(y)."""
import os
import re

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
PTX = os.path.join(os.path.dirname(HERE), "exact_attention_129_b200", "csrc", "ptx.cuh")
LOG2E = 1.4426950408889634


def constants():
    src = open(PTX).read()
    y0 = re.search(r"constexpr float kY0 = ([0-9.e+-]+)f;", src)
    m = re.search(r"constexpr float kA0 = ([0-9.e+-]+)f, kA1 = ([0-9.e+-]+)f, "
                  r"kA2 = ([0-9.e+-]+)f, kA3 = ([0-9.e+-]+)f,\s*kA4 = ([0-9.e+-]+)f;", src)
    assert y0 and m, "tanh polynomial constants not found"
    return float(y0.group(1)), [np.float32(float(v)) for v in m.groups()]


def capped_fma(s, scale, cap):
    """The kernel's steps: k1 = scale / c and K = c log2(e) in fp32 on the host,
    ka_i = K * a_i, y = s * k1, u = y * y, Horner in u, then y * P."""
    _, a = constants()
    f32 = np.float32
    k1 = f32(f32(scale) / f32(cap))
    K = f32(f32(cap) * f32(LOG2E))
    ka = [f32(K * ai) for ai in a]
    y = (np.asarray(s, np.float32) * k1).astype(np.float32)
    u = (y * y).astype(np.float32)
    p = (ka[4] * u + ka[3]).astype(np.float32)
    for k in (2, 1, 0):
        p = (p * u + ka[k]).astype(np.float32)
    return (y * p).astype(np.float32), y


@pytest.mark.parametrize("cap", [1.5, 10.0, 30.0, 50.0])
@pytest.mark.parametrize("head_dim", [64, 128, 256])
def test_relative_error_on_the_polynomial_range(cap, head_dim):
    y0, _ = constants()
    scale = head_dim ** -0.5
    smax = y0 * cap / scale
    s = np.linspace(-smax, smax, 400_001).astype(np.float32)
    got, y = capped_fma(s, scale, cap)
    y = y.astype(np.float64)
    keep = (np.abs(y) <= y0) & (y != 0)  # the kernel's own range test
    exact = cap * LOG2E * np.tanh(y[keep])
    rel = np.abs(got[keep].astype(np.float64) / exact - 1.0)
    # 1.1e-7 from the fit and its fp32 evaluation, plus the rounding of K * a_i
    assert rel.max() < 2.5e-7, rel.max()


def test_error_far_below_the_parity_bounds():
    # in the log2 domain an absolute score error e moves P by a factor 2^e; the
    # LSE bound is 1e-3 in natural-log units
    scale = 128 ** -0.5
    s = np.random.default_rng(0).normal(0, 12, 200_000).astype(np.float32)
    got, y = capped_fma(s, scale, 30.0)
    keep = np.abs(y.astype(np.float64)) <= 0.5
    exact = 30.0 * LOG2E * np.tanh(y.astype(np.float64)[keep])
    assert np.max(np.abs(got[keep] - exact)) * np.log(2) < 1e-5


def test_odd_and_zero():
    s = np.array([0.0, 1.0, -1.0, 3.0, -3.0], np.float32)
    got, _ = capped_fma(s, 0.125, 10.0)
    assert got[0] == 0.0
    assert got[1] == -got[2] and got[3] == -got[4]
