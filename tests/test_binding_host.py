"""Host logic of the Python binding, on CPU: the arguments it marshals into the
C ABI (sizes, flags, window and scale defaults, workspace sizes) and the buffer
patterns the GPU tests use.  The library is replaced by a recorder and the
CUDA-device check by a no-op, so nothing here launches or needs a GPU."""
import math

import pytest
import torch

import exact_attention_129_b200 as ea
import synth_inputs as si


class Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def f(*args):
            self.calls.append((name, args))
            return 4096 if name.endswith("workspace_size") else 0
        return f


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(ea, "library", lambda: r)
    monkeypatch.setattr(ea, "_check_cuda", lambda *ts: None)
    monkeypatch.setattr(ea, "_stream", lambda dev: None)
    return r


def _inputs(wl):
    q, k, v, do = wl.tensors()
    return q, k, v, do, torch.from_numpy(wl.cu_q), torch.from_numpy(wl.cu_k)


def test_fwd_marshals_sizes_and_defaults(rec):
    wl = si.Workload("m", [5, 0, 70], 8, 2, 128, True, lengths_k=[9, 3, 70])
    q, k, v, _, cq, ck = _inputs(wl)
    out, lse = ea.attn_fwd(q, k, v, cq, ck, wl.max_q, wl.max_k, causal=True, window=(3, None))
    name, a = rec.calls[-1]
    assert name == "attn_fwd_ex"
    # (q, k, v, cu_q, cu_k, batch, total_q, total_k, max_q, max_k, hq, hkv, d, scale,
    #  causal, window_left, window_right, softcap, return_lse, out, lse, stream)
    assert a[5:13] == (3, 75, 82, 70, 70, 8, 2, 128)
    assert math.isclose(a[13], 128 ** -0.5) and a[14] == 1
    assert a[15:19] == (3, -1, 0.0, 1)
    assert out.shape == q.shape and lse.shape == (8, 75) and lse.dtype == torch.float32


def test_fwd_split_allocates_its_workspace(rec):
    wl = si.Workload("s", [64], 4, 1, 64, False, lengths_k=[5000])
    q, k, v, _, cq, ck = _inputs(wl)
    ea.attn_fwd(q, k, v, cq, ck, 64, 5000, num_splits=6, return_lse=False)
    names = [c[0] for c in rec.calls]
    assert names[-2:] == ["attn_fwd_split_workspace_size", "attn_fwd_split"]
    a = rec.calls[-1][1]
    assert a[18] == 6 and a[19] == 0 and a[21] is None  # num_splits, return_lse, lse


def test_bwd_marshals_and_sizes_workspace(rec):
    wl = si.Workload("b", [100, 28], 4, 2, 256, False)
    q, k, v, do, cq, ck = _inputs(wl)
    out, lse = torch.zeros_like(q), torch.zeros(4, 128, dtype=torch.float32)
    ea.attn_bwd(q, k, v, out, lse, do, cq, ck, 100, 100, softcap=5.0)
    names = [c[0] for c in rec.calls]
    assert names[-2:] == ["attn_bwd_workspace_size", "attn_bwd_ex"]
    assert rec.calls[-2][1] == (2, 128, 4, 256)
    a = rec.calls[-1][1]
    # (..., batch, total_q, total_k, max_q, max_k, hq, hkv, d, scale, causal, wl, wr, cap, ...)
    assert a[8:16] == (2, 128, 128, 100, 100, 4, 2, 256)
    assert a[17:21] == (0, -1, -1, 5.0)
    assert a[25] == 4096  # the recorder's workspace size


def test_gpu_test_buffer_patterns_are_accepted(rec):
    # guarded views (a buffer with sentinel bands around the tensor) as the GPU
    # tests pass them, SplitKV with and without LSE, and the autograd path
    from tests.gpu_helpers import guarded_empty
    cpu = torch.device("cpu")
    for wl in (si.tiny(), si.Workload("r", [1, 127, 0, 515], 4, 2, 128, True)):
        q, k, v, do, cq, ck = _inputs(wl)
        for rl in (True, False):
            _, out, _ = guarded_empty(q.shape, torch.bfloat16, cpu)
            _, lse, _ = guarded_empty((wl.hq, wl.total_q), torch.float32, cpu)
            for splits in (1, 4):
                ea.attn_fwd(q, k, v, cq, ck, wl.max_q, wl.max_k, return_lse=rl, out=out,
                            lse=lse if rl else None, num_splits=splits)
        o, l = ea.attn_fwd(q, k, v, cq, ck, wl.max_q, wl.max_k, causal=True)
        grads = [guarded_empty(t.shape, torch.bfloat16, cpu)[1] for t in (q, k, v)]
        ea.attn_bwd(q, k, v, o, l, do, cq, ck, wl.max_q, wl.max_k, causal=True,
                    dq=grads[0], dk=grads[1], dv=grads[2])
        qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
        ea.attention(qg, kg, vg, cq, ck, wl.max_q, wl.max_k, causal=True).sum().backward()
        assert qg.grad is not None and qg.grad.shape == q.shape
