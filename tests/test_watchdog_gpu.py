"""Failure detection without a GPU fault.

Every wait inside the kernels is bounded.  attn_watchdog_selftest runs that same
bounded wait on a barrier nothing arrives on: it must run out, record itself in
the device error word and let the kernel exit; the host then reads the status.
Nothing traps, faults or hangs, and the context stays usable afterwards."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from tests.gpu_helpers import LSE_TOL, O_TOL, lse_err, max_abs, to_dev

pytestmark = pytest.mark.gpu

ea = pytest.importorskip("exact_attention_129_b200")


def test_bounded_wait_runs_out_and_is_reported():
    lib = ea.library()
    rc, _ = ea.last_device_error()  # start from a clear error word
    assert rc == 0
    import ctypes
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.attn_watchdog_selftest(2000, stream) == 0  # 2 ms limit
    rc, msg = ea.last_device_error()
    assert ea.STATUS[rc] == "ATTN_ERR_TIMEOUT", msg
    assert "watchdog self-test" in msg
    rc, msg = ea.last_device_error()  # reading clears the word
    assert rc == 0, msg


def test_context_usable_after_timeout():
    import ctypes
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert ea.library().attn_watchdog_selftest(1000, stream) == 0
    assert ea.last_device_error()[0] == 4
    wl = si.Workload("after_watchdog", [300, 77], 4, 2, 128, True, seed=31)
    host, (q, k, v, _), cu_q, cu_k = to_dev(wl, with_dout=False)
    out, lse = ea.attn_fwd(q, k, v, cu_q, cu_k, wl.max_q, wl.max_k, causal=True)
    rc, msg = ea.last_device_error()
    assert rc == 0, msg
    ref_o, ref_l = oracle.fwd(*host[:3], wl.cu_q, wl.cu_k, wl.scale, True)
    assert max_abs(out.float().cpu().numpy(), ref_o) <= O_TOL
    assert lse_err(lse.cpu().numpy(), ref_l) <= LSE_TOL
