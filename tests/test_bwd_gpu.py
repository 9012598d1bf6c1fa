"""GPU parity of the backward kernels (dQ, dK, dV) against the fp64 oracle."""
import pytest
import torch

import oracle
import synth_inputs as si
from tests.gpu_helpers import grad_check, guarded_empty, guards_intact, to_dev

pytestmark = pytest.mark.gpu

ea = pytest.importorskip("exact_attention_129_b200")


def run_fwd_bwd(wl, guard=True, window=None, softcap=0.0):
    host, (q, k, v, do), cu_q, cu_k = to_dev(wl)
    out, lse = ea.attn_fwd(q, k, v, cu_q, cu_k, wl.max_q, wl.max_k, scale=wl.scale,
                           causal=wl.causal, window=window, softcap=softcap, return_lse=True)
    dev = q.device
    bufs = []
    grads = []
    for like in (q, k, v):
        if guard:
            buf, view, g = guarded_empty(like.shape, torch.bfloat16, dev)
            bufs.append((buf, g))
            grads.append(view)
        else:
            grads.append(torch.empty_like(like))
    dq, dk, dv = ea.attn_bwd(q, k, v, out, lse, do, cu_q, cu_k, wl.max_q, wl.max_k,
                             scale=wl.scale, causal=wl.causal, window=window, softcap=softcap,
                             dq=grads[0], dk=grads[1], dv=grads[2])
    rc, msg = ea.last_device_error()
    assert rc == 0, msg
    for buf, g in bufs:
        assert guards_intact(buf, g), "gradient guard band overwritten"
    return host, (out, lse), (dq, dk, dv)


def check_full(wl, window=None, softcap=0.0):
    host, _, grads = run_fwd_bwd(wl, window=window, softcap=softcap)
    q, k, v, do = host
    ref = oracle.bwd(q, k, v, do, wl.cu_q, wl.cu_k, wl.scale, wl.causal, window=window,
                     softcap=softcap)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, ref):
        grad_check(g.float().cpu().numpy(), r, f"{wl.name}: {name}")


def test_tiny_config():
    check_full(si.tiny())


WINDOWS = [(0, 0), (1, 0), (63, 64), (100, 37), (-1, 17), (200, -1), (130, 0)]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_local_window(d, causal):
    for wi, win in enumerate(WINDOWS):
        wl = si.Workload(f"window{win}_d{d}", [300, 1, 515, 129], 4, 2, d, causal,
                         lengths_k=[400, 1, 515, 64], seed=40 + wi)
        check_full(wl, window=win)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("cap", [1.5, 30.0])
def test_softcap(d, cap):
    check_full(si.Workload(f"softcap{cap}_d{d}", [300, 129, 64], 4, 2, d, False, seed=51),
               softcap=cap)
    check_full(si.Workload(f"softcap{cap}_causal_d{d}", [515, 70], 4, 1, d, True, seed=52),
               softcap=cap, window=(150, 0))


RAGGED = [1, 127, 128, 129, 300, 0, 515, 64]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_ragged(d, causal):
    check_full(si.Workload(f"ragged_d{d}", RAGGED, 4, 2, d, causal, seed=13))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_gqa8_and_mha(d):
    check_full(si.Workload(f"gqa8_d{d}", [700, 260], 8, 1, d, True, seed=14))
    check_full(si.Workload(f"mha_d{d}", [333], 3, 3, d, False, seed=15))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_causal_sq_ne_sk(d):
    # bottom-right causal: some query rows see no key, some keys are seen by few rows
    wl = si.Workload(f"sq_ne_sk_d{d}", [300, 50, 200], 2, 1, d, True,
                     lengths_k=[100, 400, 200], seed=16)
    check_full(wl)


SHORT = [1, 127, 128, 0, 64, 100, 128, 33]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_direct_dq_short_segments(d, causal):
    # every key segment fits one 128-key block, so each CTA stores its rows'
    # finished dQ as bf16 (no fp32 accumulator); ragged and empty segments
    check_full(si.Workload(f"short_d{d}", SHORT, 4, 2, d, causal, seed=61))
    # s_q > s_k under bottom-right causal: rows that see no key keep dQ = 0; GQA 8/1
    check_full(si.Workload(f"short_sqsk_d{d}", [120, 128, 7], 8, 1, d, causal,
                           lengths_k=[40, 128, 100], seed=62))
    # local windows (rows whose window holds no key) and a softcap
    check_full(si.Workload(f"short_win_d{d}", [128, 90], 4, 4, d, causal,
                           lengths_k=[128, 20], seed=63), window=(5, 3))
    check_full(si.Workload(f"short_cap_d{d}", [77, 128], 4, 1, d, causal, seed=64),
               softcap=2.0)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_direct_dq_equals_accumulator_path(d, monkeypatch):
    # with one key block per segment each dQ element has exactly one partial
    # sum, so the direct bf16 store and the fp32 accumulator + convert agree bit
    # for bit; dK and dV do not depend on the choice
    wl = si.Workload(f"direct_vs_acc_d{d}", SHORT, 4, 2, d, True, seed=65)
    _, _, direct = run_fwd_bwd(wl)
    monkeypatch.setenv("ATTN_BWD_DQ_DIRECT", "0")
    _, _, acc = run_fwd_bwd(wl)
    for name, a, b in zip(("dQ", "dK", "dV"), direct, acc):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"{name} differs"


def test_keys_without_queries_get_zero_grads():
    # a segment with keys but no query rows: its dK/dV must be written as zeros
    wl = si.Workload("no_queries", [64, 0, 32], 2, 2, 128, False, lengths_k=[64, 80, 32], seed=17)
    check_full(wl)


def test_autograd_function():
    wl = si.Workload("autograd", [200, 313], 4, 2, 128, True, seed=18)
    host, (q, k, v, do), cu_q, cu_k = to_dev(wl)
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
    out = ea.attention(qg, kg, vg, cu_q, cu_k, wl.max_q, wl.max_k, causal=True)
    out.backward(do)
    ref = oracle.bwd(*host, wl.cu_q, wl.cu_k, wl.scale, True)
    for name, g, r in zip(("dQ", "dK", "dV"), (qg.grad, kg.grad, vg.grad), ref):
        grad_check(g.float().cpu().numpy(), r, f"autograd: {name}")
