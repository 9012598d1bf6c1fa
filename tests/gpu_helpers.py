"""Shared helpers for the GPU parity tests (CUDA path vs the fp64 oracle)."""
from __future__ import annotations

import numpy as np
import torch

import synth_inputs as si

# tolerances stated with the method: bf16 inputs, fp32 accumulation
O_TOL = 1e-2        # max |O - O_ref|
LSE_TOL = 1e-3      # max |LSE - LSE_ref|
GRAD_REL = 2e-2     # max |g - g_ref| <= GRAD_REL * max |g_ref|


def to_dev(wl: si.Workload, with_dout=True):
    q, k, v, do = wl.tensors(with_dout)
    dev = torch.device("cuda", 0)
    cu_q = torch.from_numpy(wl.cu_q).to(dev)
    cu_k = torch.from_numpy(wl.cu_k).to(dev)
    host = (q, k, v, do)
    devt = tuple(None if t is None else t.to(dev) for t in host)
    return host, devt, cu_q, cu_k


def guarded_empty(shape, dtype, dev, guard_elems=2048):
    """A tensor view inside a larger buffer whose guard bands hold a sentinel."""
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * guard_elems, dtype=dtype, device=dev)
    if dtype == torch.bfloat16:
        buf.view(torch.int16).fill_(0x7FC1)   # a NaN pattern nothing writes
    else:
        buf.view(torch.int32).fill_(0x7FC00001)
    view = buf[guard_elems:guard_elems + n].view(shape)
    return buf, view, guard_elems


def guards_intact(buf, guard_elems):
    if buf.dtype == torch.bfloat16:
        b = buf.view(torch.int16)
        want = 0x7FC1
    else:
        b = buf.view(torch.int32)
        want = 0x7FC00001
    return bool((b[:guard_elems] == want).all()) and bool((b[-guard_elems:] == want).all())


def max_abs(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))


def lse_err(got, ref):
    """max |LSE err| over rows; -inf must match -inf exactly."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    ninf = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), ninf), "-inf rows differ"
    if (~ninf).sum() == 0:
        return 0.0
    return float(np.max(np.abs(got[~ninf] - ref[~ninf])))
