"""CPU tests of the C ABI: the library loads, exports every declared symbol and
rejects bad arguments on the host without a GPU."""
import ctypes
import os
import re

import pytest

import exact_attention_129_b200 as ea
from exact_attention_129_b200 import build as eab

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    eab.build()
    return ea.library()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) >= {"attn_fwd", "attn_bwd", "attn_bwd_workspace_size",
                          "attn_last_device_error", "attn_version"}
    for n in names:
        assert hasattr(lib, n), n


def test_version(lib):
    assert b"sm_100a" in lib.attn_version()


def _fwd(lib, **kw):
    a = dict(q=16, k=16, v=16, cu_q=16, cu_k=16, batch=1, tq=128, tk=128, mq=128, mk=128,
             hq=4, hkv=2, d=128, scale=0.088, causal=0, rl=1, out=16, lse=16)
    a.update(kw)
    vp = ctypes.c_void_p
    return lib.attn_fwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["cu_q"]), vp(a["cu_k"]),
                        a["batch"], a["tq"], a["tk"], a["mq"], a["mk"], a["hq"], a["hkv"],
                        a["d"], a["scale"], a["causal"], a["rl"], vp(a["out"]),
                        vp(a["lse"]), None)


@pytest.mark.parametrize("bad,code", [
    (dict(d=96), 2),            # head_dim without a kernel
    (dict(d=32), 2),
    (dict(hq=3, hkv=2), 1),     # heads not a multiple
    (dict(q=8), 1),             # misaligned pointer
    (dict(out=24), 1),
    (dict(lse=0), 1),           # return_lse without an lse buffer
    (dict(batch=0), 1),
    (dict(q=0), 1),
    (dict(scale=0.0), 1),
    (dict(scale=-1.0), 1),
    (dict(scale=float("nan")), 1),
    (dict(mq=-1), 1),
])
def test_fwd_rejects_bad_arguments_without_launching(lib, bad, code):
    # every case fails in host validation, before any device call
    assert _fwd(lib, **bad) == code


@pytest.mark.parametrize("cap", [-1.0, float("nan"), float("inf")])
def test_fwd_ex_rejects_bad_softcap(lib, cap):
    # validated on the host, before any device call
    vp = ctypes.c_void_p
    rc = lib.attn_fwd_ex(vp(16), vp(16), vp(16), vp(16), vp(16), 1, 128, 128, 128, 128, 4, 2,
                         128, 0.088, 0, -1, -1, cap, 1, vp(16), vp(16), None)
    assert rc == 1
    rc = lib.attn_bwd_ex(vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), 1, 128,
                         128, 128, 128, 4, 2, 128, 0.088, 0, -1, -1, cap, vp(16), vp(16),
                         vp(16), vp(256), 1 << 30, None)
    assert rc == 1


def _fwd_split(lib, splits, ws=256, ws_bytes=1 << 30, batch=1):
    vp = ctypes.c_void_p
    return lib.attn_fwd_split(vp(16), vp(16), vp(16), vp(16), vp(16), batch, 128, 128, 128, 128,
                              4, 2, 128, 0.088, 0, -1, -1, 0.0, splits, 1, vp(16), vp(16),
                              vp(ws) if ws else None, ws_bytes, None)


@pytest.mark.parametrize("splits,kw", [
    (0, {}), (129, {}),                   # split count out of range
    (2, {"batch": 40000}),                # batch * splits beyond the grid's z limit
    (2, {"ws": 0}),                       # no workspace
    (2, {"ws": 272}),                     # workspace not 256-byte aligned
    (2, {"ws_bytes": 1024}),              # workspace too small
])
def test_fwd_split_rejects_bad_arguments(lib, splits, kw):
    assert _fwd_split(lib, splits, **kw) == 1


def test_fwd_split_workspace_size(lib):
    assert lib.attn_fwd_split_workspace_size(128, 4, 128, 0) == 0
    assert lib.attn_fwd_split_workspace_size(128, 4, 128, 129) == 0
    one = lib.attn_fwd_split_workspace_size(128, 4, 128, 1)
    four = lib.attn_fwd_split_workspace_size(128, 4, 128, 4)
    assert one >= 128 * 4 * 128 * 4 and four >= 4 * 128 * 4 * 128 * 4 and four > one


def test_bwd_rejects_small_workspace(lib):
    vp = ctypes.c_void_p
    need = lib.attn_bwd_workspace_size(1, 128, 4, 128)
    assert need > 0
    rc = lib.attn_bwd(vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), 1, 128,
                      128, 128, 128, 4, 2, 128, 0.088, 0, vp(16), vp(16), vp(16), vp(256),
                      need - 1, None)
    assert rc == 1
    rc = lib.attn_bwd(vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), 1, 128,
                      128, 128, 128, 4, 2, 128, 0.088, 0, vp(16), vp(16), vp(16), vp(100),
                      need, None)
    assert rc == 1  # workspace not 256-byte aligned


def test_workspace_size_rejects_bad_sizes(lib):
    assert lib.attn_bwd_workspace_size(0, 128, 4, 128) == 0
    assert lib.attn_bwd_workspace_size(1, 128, 0, 128) == 0


def test_python_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(ValueError):
        ea.attn_fwd(q, q, q, cu, cu, 4, 4)


def test_watchdog_selftest_rejects_bad_timeouts(lib):
    # validated on the host, before any device call
    assert lib.attn_watchdog_selftest(0, None) == 1
    assert lib.attn_watchdog_selftest(2_000_000, None) == 1


def _problem(tq=8, hq=4, tk=8, hkv=2, d=64):
    import torch
    bf = torch.bfloat16
    q = torch.zeros(tq, hq, d, dtype=bf)
    k = torch.zeros(tk, hkv, d, dtype=bf)
    v = torch.zeros(tk, hkv, d, dtype=bf)
    cq = torch.tensor([0, tq], dtype=torch.int32)
    ck = torch.tensor([0, tk], dtype=torch.int32)
    return q, k, v, cq, ck


@pytest.mark.parametrize("case", ["v_shape", "head_dim", "groups", "cu_dtype", "cu_len",
                                  "out_shape", "lse_shape", "q_rank"])
def test_python_binding_checks_shapes_before_any_launch(case):
    # the C ABI takes raw pointers: a buffer smaller than the problem would be
    # overrun on the device, so the binding rejects mismatches up front (these
    # checks run before the CUDA-device check, so they are testable on CPU)
    import torch
    q, k, v, cq, ck = _problem()
    kw = {}
    if case == "v_shape":
        v = v[:4]
    elif case == "head_dim":
        k = torch.zeros(8, 2, 128, dtype=torch.bfloat16)
        v = k.clone()
    elif case == "groups":
        k = torch.zeros(8, 3, 64, dtype=torch.bfloat16)
        v = k.clone()
    elif case == "cu_dtype":
        cq = cq.long()
    elif case == "cu_len":
        ck = torch.tensor([0, 4, 8], dtype=torch.int32)
    elif case == "out_shape":
        kw["out"] = torch.zeros(4, 4, 64, dtype=torch.bfloat16)
    elif case == "lse_shape":
        kw["lse"] = torch.zeros(8, 4, dtype=torch.float32)
    elif case == "q_rank":
        q = q.reshape(8, 256)
    with pytest.raises(ValueError) as e:
        ea.attn_fwd(q, k, v, cq, ck, 8, 8, **kw)
    assert "CUDA tensors only" not in str(e.value)


@pytest.mark.parametrize("case", ["dout_shape", "dq_shape", "dk_dtype", "lse_dtype", "missing"])
def test_python_binding_checks_backward_buffers(case):
    import torch
    q, k, v, cq, ck = _problem()
    out, dout = torch.zeros_like(q), torch.zeros_like(q)
    lse = torch.zeros(4, 8, dtype=torch.float32)
    kw = {}
    if case == "dout_shape":
        dout = dout[:2]
    elif case == "dq_shape":
        kw["dq"] = torch.zeros(8, 4, 32, dtype=torch.bfloat16)
    elif case == "dk_dtype":
        kw["dk"] = torch.zeros(8, 2, 64, dtype=torch.float32)
    elif case == "lse_dtype":
        lse = lse.double()
    elif case == "missing":
        lse = None
    with pytest.raises(ValueError) as e:
        ea.attn_bwd(q, k, v, out, lse, dout, cq, ck, 8, 8, **kw)
    assert "CUDA tensors only" not in str(e.value)
