"""GPU parity of the backward kernels (dQ, dK, dV) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from tests.gpu_helpers import GRAD_REL, guarded_empty, guards_intact, to_dev

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


def rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    if scale == 0.0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref))) / scale


def check_full(wl, window=None, softcap=0.0):
    host, _, grads = run_fwd_bwd(wl, window=window, softcap=softcap)
    q, k, v, do = host
    ref = oracle.bwd(q, k, v, do, wl.cu_q, wl.cu_k, wl.scale, wl.causal, window=window,
                     softcap=softcap)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, ref):
        gn = g.float().cpu().numpy()
        assert np.isfinite(gn).all(), f"{wl.name}: {name} not finite"
        e = rel_err(gn, r)
        assert e <= GRAD_REL, f"{wl.name}: {name} max err {e:.3e} x max|ref|"


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
    for g, r in zip((qg.grad, kg.grad, vg.grad), ref):
        assert rel_err(g.float().cpu().numpy(), r) <= GRAD_REL


def sum_properties(wl, grads, host):
    """dK summed over a segment's keys is zero (rows of dS sum to zero); dV summed
    over the keys equals dO summed over the group's query rows (rows of P sum to
    one).  Both hold at any size.

    Error bound, from the arithmetic: each dK/dV element is an fp32 tensor-core
    accumulation over n = G * ceil(s_q / 64) * 4 MMA k-steps, and those adds may
    truncate, so an element can carry a relative bias of up to n * 2^-23 (one ulp
    per add); the bias has one sign, so it adds up over the summed keys.  On top
    of it every row is rounded to bf16 once (2^-9, independent per row)."""
    _, _, _, do = host
    dq, dk, dv = (g.float().cpu() for g in grads)
    do = do.float()
    G = wl.hq // wl.hkv
    for b, (sq, sk) in enumerate(zip(wl.lengths_q, wl.lengths_k)):
        if sq == 0 or sk == 0:
            continue
        k0, q0 = int(wl.cu_k[b]), int(wl.cu_q[b])
        n_acc = G * ((sq + 63) // 64) * 4
        rel = n_acc * 2.0 ** -23
        for name, g, ref in (
            ("dK", dk[k0:k0 + sk].double(), torch.zeros(wl.hkv, wl.d, dtype=torch.float64)),
            ("dV", dv[k0:k0 + sk].double(),
             do[q0:q0 + sq].double().sum(0).view(wl.hkv, G, wl.d).sum(1)),
        ):
            tol = rel * g.abs().sum(0) + 2.0 ** -9 * np.sqrt(sk) * float(g.abs().max()) * 4
            err = (g.sum(0) - ref).abs()
            assert bool((err <= tol).all()), (
                f"segment {b}: sum {name} off by {float(err.max()):.3e} "
                f"(bound {float(tol[err.argmax() // wl.d, err.argmax() % wl.d]):.3e})")


def sampled_dq_check(wl, n_rows, seed=0):
    host, _, grads = run_fwd_bwd(wl, guard=False)
    q, k, v, do = host
    rng = np.random.default_rng(seed)
    T = wl.total_q
    rows = np.concatenate([rng.integers(0, T, size=n_rows), np.array([0, 127, 128, T - 1])])
    heads = rng.integers(0, wl.hq, size=rows.size)
    _, _, rdq = oracle.rows(q, k, v, wl.cu_q, wl.cu_k, wl.scale, wl.causal, heads, rows, dout=do)
    got = grads[0][torch.from_numpy(rows), torch.from_numpy(heads)].float().cpu().numpy()
    # the bound is relative to the largest dQ of the sampled rows' heads
    full_max = float(grads[0].float().abs().max())
    assert np.max(np.abs(got - rdq)) <= GRAD_REL * full_max
    for g in grads:
        assert torch.isfinite(g.float()).all()
    sum_properties(wl, grads, host)


def sampled_dkdv_check(wl, n_keys, kv_heads, segments, seed=0):
    """dK and dV of sampled key rows against the oracle, which computes the
    forward statistics of the chosen segments and kv groups itself."""
    host, _, grads = run_fwd_bwd(wl, guard=False)
    q, k, v, do = host
    rng = np.random.default_rng(seed)
    keys, heads = [], []
    for b in segments:
        k0, k1 = int(wl.cu_k[b]), int(wl.cu_k[b + 1])
        picks = np.concatenate([rng.integers(k0, k1, size=n_keys), [k0, k1 - 1]])
        keys.append(picks)
        heads.append(rng.choice(np.asarray(kv_heads), size=picks.size))
    keys, heads = np.concatenate(keys).astype(np.int64), np.concatenate(heads).astype(np.int32)
    rdk, rdv = oracle.cols(q, k, v, do, wl.cu_q, wl.cu_k, wl.scale, wl.causal, heads, keys)
    for got_full, ref, name in ((grads[1], rdk, "dK"), (grads[2], rdv, "dV")):
        got = got_full[torch.from_numpy(keys), torch.from_numpy(heads)].float().cpu().numpy()
        full_max = float(got_full.float().abs().max())
        err = float(np.max(np.abs(got - ref)))
        assert err <= GRAD_REL * full_max, f"{name}: {err:.3e} > {GRAD_REL} x {full_max:.3e}"


def test_full_size_varlen_gqa_sampled():
    sampled_dq_check(si.varlen_gqa(), n_rows=256)


def test_full_size_varlen_gqa_dkdv_sampled():
    wl = si.varlen_gqa()
    sampled_dkdv_check(wl, n_keys=16, kv_heads=[0, 5], segments=range(len(wl.lengths_k)))


@pytest.mark.parametrize("causal", [False, True])
def test_full_size_d256_mha_16k_dkdv_sampled(causal):
    sampled_dkdv_check(si.d256_mha(16384, causal), n_keys=24, kv_heads=[3], segments=[1])


@pytest.mark.parametrize("causal", [False, True])
def test_full_size_gqa8_128k_sampled(causal):
    sampled_dq_check(si.d256_gqa8(131072, causal), n_rows=16)


@pytest.mark.parametrize("causal", [False, True])
def test_full_size_d256_mha_16k_sampled(causal):
    sampled_dq_check(si.d256_mha(16384, causal), n_rows=32)
