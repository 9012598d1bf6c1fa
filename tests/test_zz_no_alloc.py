"""The allocation-free backward, checked against the ordinary one.

attn_bwd_static_scratch serves callers that cannot allocate device memory (a
plug-in whose host owns the allocator, a service that reserved the whole device
for its own pool, a loop that may not call cudaMalloc/cudaFree because they can
synchronise the device).  It keeps its scratch in one device array inside the
library instead of a caller-provided workspace.  This test calls it through the
C ABI several times in a row -- each call finds the previous call's leftovers
in that shared array -- and compares each result with attn_bwd on the same
inputs, within the tolerance the other backward tests use.  The file name makes
pytest collect it last.
"""
import ctypes

import pytest
import torch

import synth_inputs as si
from tests.gpu_helpers import GRAD_REL

pytestmark = pytest.mark.gpu

ea = pytest.importorskip("exact_attention_129_b200")


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_static(lib, wl, q, k, v, out, lse, do, cu_q, cu_k, dq, dk, dv):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.attn_bwd_static_scratch(
        _vp(q), _vp(k), _vp(v), _vp(out), _vp(lse), _vp(do), _vp(cu_q), _vp(cu_k),
        len(wl.lengths_q), wl.total_q, wl.total_k, wl.max_q, wl.max_k, wl.hq, wl.hkv, wl.d,
        wl.scale, int(wl.causal), _vp(dq), _vp(dk), _vp(dv), stream)


@pytest.mark.parametrize("causal", [False, True])
def test_static_scratch_matches_attn_bwd_twice(causal):
    lib = ea.library()
    dev = torch.device("cuda", 0)
    # different problems in a row, so each call starts from the previous one's
    # leftovers; the third has no key segment longer than 128, so the backward
    # stores dQ directly and only the D_i part of the array is used
    wls = [si.Workload("nsa_a", [700, 129, 64], 8, 2, 128, causal, seed=21),
           si.Workload("nsa_b", [300, 1000], 4, 1, 64, causal, seed=22),
           si.Workload("nsa_c", [100, 128, 37], 4, 2, 256, causal, seed=24)]
    for wl in wls:
        need = ea.bwd_workspace_size(len(wl.lengths_q), wl.total_q, wl.hq, wl.d)
        assert need <= (64 << 20)
        q, k, v, do = (t.to(dev) for t in wl.tensors())
        cu_q = torch.from_numpy(wl.cu_q).to(dev)
        cu_k = torch.from_numpy(wl.cu_k).to(dev)
        out, lse = ea.attn_fwd(q, k, v, cu_q, cu_k, wl.max_q, wl.max_k, causal=causal)
        ref = ea.attn_bwd(q, k, v, out, lse, do, cu_q, cu_k, wl.max_q, wl.max_k, causal=causal)
        got = tuple(torch.empty_like(t) for t in (q, k, v))
        rc = _call_static(lib, wl, q, k, v, out, lse, do, cu_q, cu_k, *got)
        assert rc == 0, ea.STATUS.get(rc, rc)
        rc, msg = ea.last_device_error()
        assert rc == 0, msg
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            err = float((g.float() - r.float()).abs().max())
            bound = GRAD_REL * float(r.float().abs().max())
            assert err <= bound, f"{wl.name} {name}: {err:.3e} > {bound:.3e}"


def test_static_scratch_rejects_problems_that_do_not_fit():
    lib = ea.library()
    dev = torch.device("cuda", 0)
    # 32768 rows x 8 heads x 128 x 4 bytes of dQ accumulator alone is 128 MiB
    wl = si.Workload("too_big", [32768], 8, 8, 128, False, seed=23)
    assert ea.bwd_workspace_size(1, wl.total_q, wl.hq, wl.d) > (64 << 20)
    x = torch.empty(16, device=dev, dtype=torch.bfloat16)
    cu = torch.tensor([0, 32768], dtype=torch.int32, device=dev)
    lse = torch.empty(16, device=dev, dtype=torch.float32)
    rc = _call_static(lib, wl, x, x, x, x, lse, x, cu, cu, x, x, x)
    assert ea.STATUS[rc] == "ATTN_ERR_SCRATCH_TOO_SMALL"
