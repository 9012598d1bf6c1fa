"""GPU parity of the forward kernel against the fp64 oracle (O and LSE)."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from tests.gpu_helpers import LSE_TOL, check_o, guarded_empty, guards_intact, lse_err, to_dev

pytestmark = pytest.mark.gpu

ea = pytest.importorskip("exact_attention_129_b200")


def run_fwd(wl, return_lse=True, guard=True, window=None, softcap=0.0, num_splits=1):
    host, (q, k, v, _), cu_q, cu_k = to_dev(wl, with_dout=False)
    dev = q.device
    obuf, out, og = guarded_empty(q.shape, torch.bfloat16, dev)
    lbuf, lse, lg = guarded_empty((wl.hq, wl.total_q), torch.float32, dev)
    ea.attn_fwd(q, k, v, cu_q, cu_k, wl.max_q, wl.max_k, scale=wl.scale, causal=wl.causal,
                window=window, softcap=softcap, return_lse=return_lse, out=out,
                lse=lse if return_lse else None, num_splits=num_splits)
    rc, msg = ea.last_device_error()
    assert rc == 0, msg
    assert guards_intact(obuf, og), "out guard band overwritten"
    assert guards_intact(lbuf, lg), "lse guard band overwritten"
    return host, out, lse


def check_full(wl, window=None, softcap=0.0, num_splits=1):
    host, out, lse = run_fwd(wl, window=window, softcap=softcap, num_splits=num_splits)
    q, k, v, _ = host
    ref_o, ref_lse = oracle.fwd(q, k, v, wl.cu_q, wl.cu_k, wl.scale, wl.causal, window=window,
                                softcap=softcap)
    # the same attention over |V| gives the P-rounding part of the O bound
    ref_pabsv, _ = oracle.fwd(q, k, v.float().abs(), wl.cu_q, wl.cu_k, wl.scale, wl.causal,
                              window=window, softcap=softcap)
    eo = check_o(out.float().cpu().numpy(), ref_o, ref_pabsv, wl.name)[0]
    el = lse_err(lse.cpu().numpy(), ref_lse)
    assert el <= LSE_TOL, f"{wl.name}: max |LSE err| {el:.3e}"
    return eo, el


def test_tiny_config():
    check_full(si.tiny())


RAGGED = [1, 127, 128, 129, 300, 0, 515, 64]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_ragged(d, causal):
    check_full(si.Workload(f"ragged_d{d}", RAGGED, 4, 2, d, causal, seed=3))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_gqa8_and_mqa(d):
    check_full(si.Workload(f"gqa8_d{d}", [700, 260], 8, 1, d, True, seed=4))
    check_full(si.Workload(f"mha_d{d}", [333], 3, 3, d, False, seed=5))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_causal_sq_ne_sk(d):
    # bottom-right causal; the first segment has query rows that see no key
    wl = si.Workload(f"sq_ne_sk_d{d}", [300, 50, 200], 2, 1, d, True,
                     lengths_k=[100, 400, 200], seed=6)
    check_full(wl)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_lse_flag_does_not_change_out(d):
    wl = si.Workload(f"lseflag_d{d}", [1000, 24], 4, 4, d, False, seed=7)
    _, o1, _ = run_fwd(wl, return_lse=True)
    _, o2, _ = run_fwd(wl, return_lse=False)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_epilogue_after_last_pv(d, monkeypatch):
    """The softmax warps reach their final wait only after the tile's last P.V
    has completed (the test hook holds them 200 us).  A parity wait on the
    per-P.V barrier would then name a phase two behind and never return; the
    single-phase final barrier must let every tile finish."""
    monkeypatch.setenv("ATTN_TEST_EPILOGUE_DELAY_US", "200")
    for causal in (False, True):
        check_full(si.Workload(f"late_epilogue_d{d}", [1000, 257, 96], 4, 2, d, causal, seed=9))


# local (sliding-window) masks: bounds below, at and above the block sizes,
# one-sided windows, and segments with s_q != s_k
WINDOWS = [(0, 0), (1, 0), (63, 64), (100, 37), (-1, 17), (200, -1), (130, 0)]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_local_window(d, causal):
    for wi, win in enumerate(WINDOWS):
        wl = si.Workload(f"window{win}_d{d}", [300, 1, 515, 129], 4, 2, d, causal,
                         lengths_k=[400, 1, 515, 64], seed=20 + wi)
        check_full(wl, window=win)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("cap", [1.5, 30.0])
def test_softcap(d, cap):
    check_full(si.Workload(f"softcap{cap}_d{d}", [300, 129, 64], 4, 2, d, False, seed=31),
               softcap=cap)
    wl = si.Workload(f"softcap{cap}_causal_d{d}", [515, 70], 4, 1, d, True, seed=32)
    check_full(wl, softcap=cap, window=(150, 0))


# SplitKV: short query segments against long key segments, split counts from 1
# to more than there are key blocks (the extra splits see no key)
DECODE = dict(lengths_q=[1, 3, 64, 130], lengths_k=[2000, 5000, 300, 1024])


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("splits", [1, 2, 3, 7, 64, 128])
def test_splitkv(d, splits):
    for causal in (False, True):
        wl = si.Workload(f"decode_d{d}_s{splits}", DECODE["lengths_q"], 8, 2, d, causal,
                         lengths_k=DECODE["lengths_k"], seed=60)
        check_full(wl, num_splits=splits)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_splitkv_window_softcap_no_lse(d):
    wl = si.Workload(f"decode_mask_d{d}", DECODE["lengths_q"], 4, 1, d, True,
                     lengths_k=DECODE["lengths_k"], seed=61)
    check_full(wl, num_splits=5, window=(700, 0), softcap=20.0)
    # return_lse off: O must not change
    _, o1, _ = run_fwd(wl, num_splits=5, window=(700, 0), softcap=20.0)
    _, o2, _ = run_fwd(wl, return_lse=False, num_splits=5, window=(700, 0), softcap=20.0)
    assert torch.equal(o1, o2)


# packed GQA: the G query heads of a key/value head share the tile rows
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("group", [2, 4, 8, 16])
def test_pack_gqa_forced(d, group, monkeypatch):
    monkeypatch.setenv("ATTN_PACK_GQA", "1")
    hkv = 2 if group <= 8 else 1
    for causal in (False, True):
        wl = si.Workload(f"pack_g{group}_d{d}", [300, 1, 515, 129], group * hkv, hkv, d, causal,
                         lengths_k=[400, 1, 515, 64], seed=70 + group)
        check_full(wl)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_pack_gqa_masks_and_splits(d, monkeypatch):
    monkeypatch.setenv("ATTN_PACK_GQA", "1")
    wl = si.Workload(f"pack_mask_d{d}", [77, 200, 5], 8, 2, d, True, lengths_k=[900, 200, 3000],
                     seed=80)
    check_full(wl, window=(300, 0), softcap=10.0)
    check_full(wl, num_splits=4, window=(300, 0))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_unpacked_forced(d, causal, monkeypatch):
    # GQA packs by default; one query head per tile stays correct when forced
    monkeypatch.setenv("ATTN_PACK_GQA", "0")
    check_full(si.Workload(f"unpacked_ragged_d{d}", RAGGED, 4, 2, d, causal, seed=82))
    wl = si.Workload(f"unpacked_window_d{d}", [300, 1, 515, 129], 8, 1, d, causal,
                     lengths_k=[400, 1, 515, 64], seed=83)
    check_full(wl, window=(100, 37))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_decode_shapes_default_path(d):
    # short query segments with G = 4 (packed by default), with and without SplitKV
    wl = si.Workload(f"decode_small_d{d}", [1, 16, 100], 8, 2, d, True,
                     lengths_k=[3000, 700, 4100], seed=81)
    for splits in (1, 6):
        check_full(wl, num_splits=splits)


def test_deterministic():
    wl = si.Workload("det", [777, 1500], 4, 2, 128, True, seed=8)
    outs = [run_fwd(wl)[1:] for _ in range(3)]
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


def test_large_scores_stay_finite():
    # scale 1 on N(0, 4) inputs: scores of order +-100 exercise the running-max rescale
    wl = si.Workload("large", [640], 2, 2, 128, False, seed=9)
    host, (q, k, v, _), cu_q, cu_k = to_dev(wl, with_dout=False)
    q2, k2 = (q.float() * 2).bfloat16(), (k.float() * 2).bfloat16()
    out, lse = ea.attn_fwd(q2, k2, v, cu_q, cu_k, wl.max_q, wl.max_k, scale=1.0)
    ref_o, ref_l = oracle.fwd(q2.cpu(), k2.cpu(), host[2], wl.cu_q, wl.cu_k, 1.0, False)
    # rows this peaked are dominated by one or two keys: the per-element bound
    # from the bf16 rounding of P and O applies
    ref_pabsv, _ = oracle.fwd(q2.cpu(), k2.cpu(), host[2].float().abs(), wl.cu_q, wl.cu_k, 1.0,
                              False)
    check_o(out.float().cpu().numpy(), ref_o, ref_pabsv, wl.name)
    # |LSE| ~ 100 here: allow the same relative error as at |LSE| ~ 1
    assert lse_err(lse.cpu().numpy(), ref_l) <= LSE_TOL * max(1.0, np.abs(ref_l).max() / 10)


# The forward's grid: persistent CTAs (one per SM, each walking a static share
# of the tiles, the barrier phases running on from tile to tile) for equal
# segments without key bounds, one CTA per tile otherwise.  Each mode forced on
# the other's workloads: ragged and empty segments, masks, windows, softcap,
# SplitKV, and more tiles than CTAs so each CTA walks several.
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("grid", ["persistent", "tiles"])
def test_grid_modes_forced(d, grid, monkeypatch):
    monkeypatch.setenv("ATTN_FWD_GRID", grid)
    check_full(si.Workload(f"grid_{grid}_ragged_d{d}", RAGGED, 4, 2, d, True, seed=90))
    check_full(si.Workload(f"grid_{grid}_dense_d{d}", [1024] * 6, 8, 8, d, False, seed=91))
    wl = si.Workload(f"grid_{grid}_window_d{d}", [300, 1, 515, 129, 0, 700], 8, 1, d, True,
                     lengths_k=[400, 1, 515, 64, 9, 700], seed=92)
    check_full(wl, window=(100, 37), softcap=20.0)
    check_full(wl, num_splits=3)


# The two-CTA forward (cta_group::2 MMAs over a CTA pair) is the default at
# head_dim 256 and opt-in at 128; each head_dim forced both ways on ragged,
# causal, windowed and packed-GQA workloads
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("pair", ["0", "1"])
def test_cta_pair_forced(d, pair, monkeypatch):
    monkeypatch.setenv("ATTN_FWD_PAIR", pair)
    check_full(si.Workload(f"pair{pair}_ragged_d{d}", RAGGED, 4, 2, d, True, seed=95))
    check_full(si.Workload(f"pair{pair}_mha_d{d}", [777, 300], 3, 3, d, False, seed=96))
    wl = si.Workload(f"pair{pair}_window_d{d}", [300, 1, 515, 129], 8, 1, d, True,
                     lengths_k=[400, 1, 515, 64], seed=97)
    check_full(wl, window=(100, 37))
