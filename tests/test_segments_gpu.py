"""A packed varlen batch on the GPU equals independent calls of its segments.

Every tile (forward) and every key block (backward) depends only on its own
segment: rows and keys past a segment's end are masked, and a masked P is an
exact zero.  So the forward's O and LSE and the backward's dK and dV of each
segment must equal, bit for bit, those of the same segment run as a batch of
one (whose grid, persistent or not, and tile count differ).  dQ sums fp32
partials of several key blocks with atomic adds, in an order that varies, so
it is left to the oracle comparisons of the other files.
"""
import pytest
import torch

import synth_inputs as si

pytestmark = pytest.mark.gpu

ea = pytest.importorskip("exact_attention_129_b200")

LENGTHS = [300, 1, 515, 129, 0, 64, 1000]


def run(q, k, v, do, lengths, hq, causal, scale):
    dev = q.device
    cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0).tolist()), dtype=torch.int32,
                      device=dev)
    mx = max(lengths)
    out, lse = ea.attn_fwd(q, k, v, cu, cu, mx, mx, scale=scale, causal=causal, return_lse=True)
    dq, dk, dv = ea.attn_bwd(q, k, v, out, lse, do, cu, cu, mx, mx, scale=scale, causal=causal)
    rc, msg = ea.last_device_error()
    assert rc == 0, msg
    return out, lse, dk, dv


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_batch_equals_segments(d, causal):
    wl = si.Workload(f"segments_d{d}", LENGTHS, 8, 2, d, causal, seed=98)
    q, k, v, do = (t.to(torch.device("cuda", 0)) for t in wl.tensors())
    out, lse, dk, dv = run(q, k, v, do, LENGTHS, wl.hq, causal, wl.scale)
    r0 = 0
    for s in LENGTHS:
        if s > 0:
            sl = slice(r0, r0 + s)
            o1, l1, dk1, dv1 = run(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(),
                                   do[sl].contiguous(), [s], wl.hq, causal, wl.scale)
            assert torch.equal(out[sl], o1), f"d{d} segment of {s}: O"
            assert torch.equal(lse[:, sl], l1), f"d{d} segment of {s}: LSE"
            assert torch.equal(dk[sl], dk1), f"d{d} segment of {s}: dK"
            assert torch.equal(dv[sl], dv1), f"d{d} segment of {s}: dV"
        r0 += s
