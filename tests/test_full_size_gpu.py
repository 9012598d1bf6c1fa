"""Full-size GPU parity: every stated workload at its full size, run forward and
backward once in the launch configuration the bench times, checked against the
fp64 oracle on outputs the oracle computes one by one.

Per workload:
  * O, LSE and dQ of sampled query rows (random rows plus the edge rows of each
    segment), each computed by the oracle from that row's own scores;
  * under a causal mask, rows 0-3 of every segment for every query head: the
    rows that see one to four keys, where bf16 rounding does not average out;
  * dK and dV of sampled key rows (``oracle.cols``).  Without a mask a key row
    depends on every query row of its group, so this runs where the oracle
    finishes in seconds (up to 8K keys per segment); under a causal mask the
    keys come from the last positions of a segment, which only the last rows
    see, so it runs at every length, 128K included;
  * the two sum identities of dK and dV, which hold at any size.

Bounds: O per element by ``o_bound`` (the stated 1e-2 wherever bf16 arithmetic
can reach it), LSE 1e-3, gradients 2e-2 times the largest magnitude among the
oracle's values for the same outputs.  No bound takes its scale from the GPU's
own output.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from tests.gpu_helpers import LSE_TOL, check_o, grad_check, lse_err

pytestmark = pytest.mark.gpu

ea = pytest.importorskip("exact_attention_129_b200")

_CACHE = {}


def host_tensors(wl):
    """bf16 CPU tensors and their float64 copies, kept for the next workload of
    the same shape (causal and non-causal variants share their inputs)."""
    key = (wl.total_q, wl.total_k, wl.hq, wl.hkv, wl.d, wl.seed)
    if key not in _CACHE:
        _CACHE.clear()
        bf = wl.tensors()
        f64 = tuple(np.ascontiguousarray(t.to(torch.float64).numpy()) for t in bf)
        _CACHE[key] = (bf, f64)
    return _CACHE[key]


def run_device(wl, bf, fwd_only=False):
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in bf)
    cu_q = torch.from_numpy(wl.cu_q).to(dev)
    cu_k = torch.from_numpy(wl.cu_k).to(dev)
    out, lse = ea.attn_fwd(q, k, v, cu_q, cu_k, wl.max_q, wl.max_k, scale=wl.scale,
                           causal=wl.causal, return_lse=True)
    grads = None
    if not fwd_only:
        grads = ea.attn_bwd(q, k, v, out, lse, do, cu_q, cu_k, wl.max_q, wl.max_k,
                            scale=wl.scale, causal=wl.causal)
    torch.cuda.synchronize()
    rc, msg = ea.last_device_error()
    assert rc == 0, msg
    del q, k, v, do
    return out, lse, grads


def sample_rows(wl, n_random, rng, few_key_sweep):
    """(rows, heads): random (row, head) pairs, the edge rows of up to eight
    segments, and with ``few_key_sweep`` rows 0-3 of every segment for every head."""
    T = wl.total_q
    rows = [rng.integers(0, T, size=n_random)]
    heads = [rng.integers(0, wl.hq, size=n_random)]
    for b in range(min(8, len(wl.lengths_q))):
        s, r0 = wl.lengths_q[b], int(wl.cu_q[b])
        edge = np.array([o for o in (0, 1, 127, 128, 129, s - 1) if 0 <= o < s]) + r0
        rows.append(edge)
        heads.append(rng.integers(0, wl.hq, size=edge.size))
    if few_key_sweep:
        for b, s in enumerate(wl.lengths_q):
            r = np.arange(min(4, s)) + int(wl.cu_q[b])
            rows.append(np.repeat(r, wl.hq))
            heads.append(np.tile(np.arange(wl.hq), r.size))
    return np.concatenate(rows).astype(np.int64), np.concatenate(heads).astype(np.int32)


def sum_properties(wl, grads, dout):
    """dK summed over a segment's keys is zero (rows of dS sum to zero); dV summed
    over the keys equals dO summed over the group's query rows (rows of P sum to
    one).  Both hold at any size.

    Error bound, from the arithmetic: each dK/dV element is an fp32 tensor-core
    accumulation over n = G * ceil(s_q / 64) * 4 MMA k-steps, and those adds may
    truncate, so an element can carry a relative bias of up to n * 2^-23 (one ulp
    per add); the bias has one sign, so it adds up over the summed keys.  On top
    of it every row is rounded to bf16 once (2^-9, independent per row)."""
    dk, dv = (g.float().cpu() for g in grads[1:])
    do = torch.from_numpy(dout)
    G = wl.hq // wl.hkv
    for b, (sq, sk) in enumerate(zip(wl.lengths_q, wl.lengths_k)):
        if sq == 0 or sk == 0:
            continue
        k0, q0 = int(wl.cu_k[b]), int(wl.cu_q[b])
        rel = G * ((sq + 63) // 64) * 4 * 2.0 ** -23
        for name, g, ref in (
            ("dK", dk[k0:k0 + sk].double(), torch.zeros(wl.hkv, wl.d, dtype=torch.float64)),
            ("dV", dv[k0:k0 + sk].double(), do[q0:q0 + sq].sum(0).view(wl.hkv, G, wl.d).sum(1)),
        ):
            tol = rel * g.abs().sum(0) + 2.0 ** -9 * np.sqrt(sk) * float(g.abs().max()) * 4
            err = (g.sum(0) - ref).abs()
            assert bool((err <= tol).all()), (
                f"{wl.name} segment {b}: sum {name} off by {float(err.max()):.3e}")


def key_sample(wl, n_keys, rng, tail):
    """(keys, kv heads).  With ``tail``: keys from the last ``tail`` positions of
    up to four segments, on the first and the last kv head; without (every query
    row of the group sees every key): keys over the whole of up to two segments,
    on the last kv head, so that the oracle's forward statistics stay small."""
    keys, heads = [], []
    kv_choice = [0, wl.hkv - 1] if tail else [wl.hkv - 1]
    for b in range(min(4 if tail else 2, len(wl.lengths_k))):
        k0, k1 = int(wl.cu_k[b]), int(wl.cu_k[b + 1])
        if k1 <= k0:
            continue
        lo = max(k0, k1 - tail) if tail else k0
        picks = np.concatenate([rng.integers(lo, k1, size=n_keys), [lo, k1 - 1]])
        keys.append(picks)
        heads.append(rng.choice(kv_choice, size=picks.size))
    return np.concatenate(keys).astype(np.int64), np.concatenate(heads).astype(np.int32)


def full_size_check(wl, n_rows, dkdv, record_property, fwd_only=False, seed=0):
    """``dkdv``: None, or (keys per segment, tail length or 0 for the whole segment)."""
    bf, (q, k, v, do) = host_tensors(wl)
    out, lse, grads = run_device(wl, bf, fwd_only)
    rng = np.random.default_rng(seed)
    rows, heads = sample_rows(wl, n_rows, rng, few_key_sweep=wl.causal)
    ro, rl, rdq = oracle.rows(q, k, v, wl.cu_q, wl.cu_k, wl.scale, wl.causal, heads, rows,
                              dout=None if fwd_only else do)
    rpv, _, _ = oracle.rows(q, k, np.abs(v), wl.cu_q, wl.cu_k, wl.scale, wl.causal, heads, rows)
    r_t, h_t = torch.from_numpy(rows), torch.from_numpy(heads)
    eo, eo_strict, n_above = check_o(out[r_t, h_t].float().cpu().numpy(), ro, rpv, wl.name)
    el = lse_err(lse[h_t, r_t].cpu().numpy(), rl)
    assert el <= LSE_TOL, f"{wl.name}: max |LSE err| {el:.3e}"
    record_property("o_err_max", eo)
    record_property("o_err_max_where_bound_is_1e-2", eo_strict)
    record_property("o_elems_above_1e-2", n_above)
    record_property("lse_err_max", el)
    if fwd_only:
        return
    record_property("dq_rel", grad_check(grads[0][r_t, h_t].float().cpu().numpy(), rdq,
                                         f"{wl.name}: dQ"))
    for g in grads:
        assert bool(torch.isfinite(g).all())
    if dkdv is not None:
        n_keys, tail = dkdv
        keys, kh = key_sample(wl, n_keys, rng, tail)
        rdk, rdv = oracle.cols(q, k, v, do, wl.cu_q, wl.cu_k, wl.scale, wl.causal, kh, keys)
        k_t, kh_t = torch.from_numpy(keys), torch.from_numpy(kh)
        record_property("dk_rel", grad_check(grads[1][k_t, kh_t].float().cpu().numpy(), rdk,
                                             f"{wl.name}: dK"))
        record_property("dv_rel", grad_check(grads[2][k_t, kh_t].float().cpu().numpy(), rdv,
                                             f"{wl.name}: dV"))
    sum_properties(wl, grads, do)


# (workload, sampled random rows, dK/dV keys: (keys per segment, tail or 0) or None).
# Ordered so that workloads with the same inputs run back to back.
TAIL = 256
CASES = [
    ("varlen_gqa", si.varlen_gqa, 192, (12, 0)),
    ("gqa_1k", lambda: si.single_gqa(1024), 64, (16, 0)),
    ("gqa_4k", lambda: si.single_gqa(4096), 64, (16, 0)),
    ("gqa_16k", lambda: si.single_gqa(16384), 48, None),
    ("gqa_16k_causal", lambda: si.single_gqa(16384, True), 48, (16, TAIL)),
    ("gqa_32k", lambda: si.single_gqa(32768), 32, None),
    ("gqa_64k", lambda: si.single_gqa(65536), 24, None),
] + [
    (f"d256_mha_{s // 1024}k{'_causal' if c else ''}", (lambda s=s, c=c: si.d256_mha(s, c)),
     32 if s <= 32768 else 16, (12, TAIL) if c else ((8, 0) if s <= 8192 else None))
    for s in (4096, 8192, 16384, 32768, 65536, 131072) for c in (False, True)
] + [
    ("d256_gqa8_128k", lambda: si.d256_gqa8(131072, False), 16, None),
    ("d256_gqa8_128k_causal", lambda: si.d256_gqa8(131072, True), 16, (12, TAIL)),
]


@pytest.mark.parametrize("name,make,n_rows,dkdv", CASES, ids=[c[0] for c in CASES])
def test_full_size(name, make, n_rows, dkdv, record_property):
    full_size_check(make(), n_rows, dkdv, record_property)


def test_full_size_d64_forward(record_property):
    # the head_dim-64 workload is forward only
    full_size_check(si.d64_mha(), 128, None, record_property, fwd_only=True)
