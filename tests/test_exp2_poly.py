"""CPU check of the FMA-pipe exp2 used by the forward softmax.

The kernel's constants are read from ptx.cuh and its fp32 steps are replayed
with numpy (round-to-nearest fp32 at every step, as the GPU does), then the
result is compared with the exact 2^x over the whole argument range the
softmax can produce (the running max is stale by at most 8, so x <= 8;
masked scores are -inf)."""
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
PTX = os.path.join(os.path.dirname(HERE), "exact_attention_129_b200", "csrc", "ptx.cuh")


def constants():
    src = open(PTX).read()
    m = re.search(r"constexpr float kC0 = ([0-9.e+-]+)f, kC1 = ([0-9.e+-]+)f, "
                  r"kC2 = ([0-9.e+-]+)f, kC3 = ([0-9.e+-]+)f;", src)
    assert m, "exp2 polynomial constants not found"
    return [np.float32(float(v)) for v in m.groups()]


def exp2_fma(x):
    c0, c1, c2, c3 = constants()
    f32 = np.float32
    x = np.maximum(np.asarray(x, np.float32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(np.float32)
    n = (t - f32(12582912.0)).astype(np.float32)
    f = (n * f32(-1.0) + x).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64),
                        np.arange(-125, 9, dtype=np.float64) + 0.5,
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    got = exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    # degree-3 minimax error 7.5e-5 plus a few fp32 roundings
    assert rel.max() < 1.0e-4, rel.max()


def test_masked_and_tiny_arguments():
    got = exp2_fma(np.array([-np.inf, -1000.0, -126.0, -125.0], np.float32))
    assert np.all(np.isfinite(got))
    assert np.all(got <= np.float32(2.0 ** -124))
    assert np.all(got > 0)


def test_error_far_below_bf16_resolution():
    # the P that feeds the P.V product is rounded to bf16 (2^-9 relative)
    x = np.random.default_rng(0).uniform(-30, 8, 100_000).astype(np.float32)
    rel = np.abs(exp2_fma(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 2.0 ** -9 / 10
