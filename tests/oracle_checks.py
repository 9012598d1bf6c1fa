"""Pins for the fp64 oracle: checks against facts that do not come from the oracle.

Each ``check_*`` returns ``(ok, message)`` so the same battery can (a) pass on
the oracle the suite trusts and (b) be shown to fail on copies of the oracle
with one planted mistake.  The facts used:

* brute-force central finite differences of L = sum(dO * O) (pins the whole
  backward against the forward);
* an independent fp64 torch implementation (explicit mask + softmax + matmul,
  gradients by autograd) -- the special case "library routine";
* scipy's logsumexp over explicitly computed scores;
* closed forms: constant V gives O = V; Q = 0 gives the mean of the allowed
  values and LSE = log(#allowed); a causal row 0 sees only key 0; a single key
  gives O = v_0; shifting every key of a segment by one vector leaves O
  unchanged and moves LSE_i by scale * <q_i, shift>;
* gradient identities: sum_j dK_j = 0 (each row of dS sums to zero) and
  sum_j dV_j = sum over the group's rows of dO (each row of P sums to one);
* structure: a packed varlen batch equals independent dense calls, and GQA
  equals MHA with K/V repeated per group (dK/dV then sum over the group);
* local masks and the softcap: window (0, 0) leaves one key (O = v_j, LSE = the
  capped score, a closed form); a window wider than the segment is no window;
  (-1, 0) is causal; a huge cap is no cap; a windowed row equals unmasked
  attention over its key slice; plus the torch reference and finite
  differences on windowed and capped cases.
"""
from __future__ import annotations

import numpy as np
import torch
from scipy.special import logsumexp

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(shape, seed):
    return _rng(seed).standard_normal(shape)


def _cu(lengths):
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(lengths)
    return cu


def _close(a, b, tol):
    a, b = np.asarray(a), np.asarray(b)
    fin = np.isfinite(b)
    if not np.array_equal(np.isfinite(a), fin):
        return False, "finite pattern differs"
    if not np.array_equal(a[~fin], b[~fin]):
        return False, "non-finite values differ"
    if fin.sum() == 0:
        return True, "ok"
    err = float(np.max(np.abs(a[fin] - b[fin])))
    scale = max(1.0, float(np.max(np.abs(b[fin]))))
    return (err <= tol * scale), f"max err {err:.3e} (tol {tol:.1e} x {scale:.2e})"


# --------------------------------------------------------------------------
# independent torch fp64 implementation (explicit mask, autograd)
# --------------------------------------------------------------------------
def torch_reference(q, k, v, dout, lengths_q, lengths_k, scale, causal, window=None,
                    softcap=0.0):
    """Dense per-segment softmax(scale QK^T + mask) V with autograd (fp64 CPU).

    ``window`` (left, right) and ``softcap`` follow the reading stated in the
    oracle's header: inclusive key distances around the bottom-right diagonal,
    and c * tanh(s / c) of the scaled score; autograd supplies the derivatives."""
    tq = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    outs, lses = [], []
    oq = ok_ = 0
    for sq, sk in zip(lengths_q, lengths_k):
        qs = tq[oq:oq + sq].permute(1, 0, 2)                      # [Hq, sq, D]
        ks = tk[ok_:ok_ + sk].permute(1, 0, 2).repeat_interleave(G, 0)
        vs = tv[ok_:ok_ + sk].permute(1, 0, 2).repeat_interleave(G, 0)
        s = scale * qs @ ks.transpose(1, 2)                       # [Hq, sq, sk]
        if softcap and softcap > 0:
            s = softcap * torch.tanh(s / softcap)
        i = torch.arange(sq).view(-1, 1)
        j = torch.arange(sk).view(1, -1)
        diag = i + (sk - sq)
        allowed = (j <= diag) if causal else torch.ones(sq, sk, dtype=torch.bool)
        if window is not None and window[0] >= 0:
            allowed = allowed & (j >= diag - window[0])
        if window is not None and window[1] >= 0:
            allowed = allowed & (j <= diag + window[1])
        s = s.masked_fill(~allowed, float("-inf"))
        lse = torch.logsumexp(s, dim=-1)                          # [Hq, sq]
        p = torch.exp(s - lse.unsqueeze(-1))
        p = torch.nan_to_num(p, nan=0.0)
        outs.append((p @ vs).permute(1, 0, 2))
        lses.append(lse)
        oq += sq
        ok_ += sk
    out = torch.cat(outs, 0)
    lse = torch.cat(lses, 1)
    grads = (None, None, None)
    if dout is not None:
        (out * torch.tensor(dout, dtype=torch.float64)).sum().backward()
        grads = tuple(t.grad.numpy() if t.grad is not None else np.zeros(t.shape)
                      for t in (tq, tk, tv))
    return out.detach().numpy(), lse.detach().numpy(), grads


# --------------------------------------------------------------------------
# the battery
# --------------------------------------------------------------------------
CASES = [
    # (lengths_q, lengths_k, Hq, Hkv, D, causal)
    ([7], [7], 2, 1, 4, False),
    ([7], [7], 2, 1, 4, True),
    ([3, 5], [3, 5], 2, 2, 8, True),
    ([4, 6], [6, 3], 4, 2, 4, True),      # s_q != s_k, bottom-right causal
    ([5, 0, 4], [5, 0, 4], 2, 1, 4, False),  # a zero-length segment
]


def check_finite_differences(mutation=0, eps=1e-6, tol=1e-6):
    for ci, (lq, lk, Hq, Hkv, D, causal) in enumerate(CASES):
        Tq, Tk = sum(lq), sum(lk)
        q = _rand((Tq, Hq, D), 10 + ci)
        k = _rand((Tk, Hkv, D), 20 + ci)
        v = _rand((Tk, Hkv, D), 30 + ci)
        do = _rand((Tq, Hq, D), 40 + ci)
        scale = 0.7
        cq, ck = _cu(lq), _cu(lk)
        dq, dk, dv = oracle.bwd(q, k, v, do, cq, ck, scale, causal, mutation=mutation)

        def loss(q_, k_, v_):
            o, _ = oracle.fwd(q_, k_, v_, cq, ck, scale, causal, mutation=mutation)
            return float(np.sum(o * do))

        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            flat = x.reshape(-1)
            for t in range(flat.size):
                old = flat[t]
                flat[t] = old + eps
                lp = loss(q, k, v)
                flat[t] = old - eps
                lm = loss(q, k, v)
                flat[t] = old
                num.reshape(-1)[t] = (lp - lm) / (2 * eps)
            ok, msg = _close(g, num, tol)
            if not ok:
                return False, f"FD case {ci} d{name}: {msg}"
    return True, "ok"


def check_torch_reference(mutation=0, tol=1e-12):
    for ci, (lq, lk, Hq, Hkv, D, causal) in enumerate(CASES):
        Tq, Tk = sum(lq), sum(lk)
        q = _rand((Tq, Hq, D), 50 + ci)
        k = _rand((Tk, Hkv, D), 60 + ci)
        v = _rand((Tk, Hkv, D), 70 + ci)
        do = _rand((Tq, Hq, D), 80 + ci)
        scale = D ** -0.5
        cq, ck = _cu(lq), _cu(lk)
        o, lse = oracle.fwd(q, k, v, cq, ck, scale, causal, mutation=mutation)
        dq, dk, dv = oracle.bwd(q, k, v, do, cq, ck, scale, causal, mutation=mutation)
        ro, rlse, (rdq, rdk, rdv) = torch_reference(q, k, v, do, lq, lk, scale, causal)
        for name, a, b in (("O", o, ro), ("LSE", lse, rlse), ("dQ", dq, rdq),
                           ("dK", dk, rdk), ("dV", dv, rdv)):
            ok, msg = _close(a, b, tol)
            if not ok:
                return False, f"torch case {ci} {name}: {msg}"
    return True, "ok"


def check_lse_logsumexp(mutation=0):
    lq = [9, 16]
    Hq, Hkv, D = 4, 2, 8
    q = 3 * _rand((25, Hq, D), 1)      # large scores: the max term matters
    k = 3 * _rand((25, Hkv, D), 2)
    v = _rand((25, Hkv, D), 3)
    for causal in (False, True):
        _, lse = oracle.fwd(q, k, v, _cu(lq), _cu(lq), 0.5, causal, mutation=mutation)
        off = 0
        for s in lq:
            for h in range(Hq):
                hk = h // (Hq // Hkv)
                sc = 0.5 * q[off:off + s, h] @ k[off:off + s, hk].T
                if causal:
                    sc = np.where(np.tri(s, s, 0, dtype=bool), sc, -np.inf)
                ref = logsumexp(sc, axis=1)
                ok, msg = _close(lse[h, off:off + s], ref, 1e-12)
                if not ok:
                    return False, f"logsumexp causal={causal} h={h}: {msg}"
            off += s
    return True, "ok"


def check_closed_forms(mutation=0):
    Hq, Hkv, D = 4, 2, 8
    lq = [6, 11]
    cu = _cu(lq)
    T = sum(lq)
    q = _rand((T, Hq, D), 4)
    k = _rand((T, Hkv, D), 5)
    # constant V -> O = V
    c = _rand((1, Hkv, D), 6)
    vconst = np.repeat(c, T, axis=0)
    for causal in (False, True):
        o, _ = oracle.fwd(q, k, vconst, cu, cu, 0.9, causal, mutation=mutation)
        G = Hq // Hkv
        ref = np.repeat(c, G, axis=1).repeat(T, axis=0)
        ok, msg = _close(o, ref, 1e-12)
        if not ok:
            return False, f"constant V causal={causal}: {msg}"
    # causal row 0 sees only key 0: O_0 = v_0, LSE_0 = s_00
    v = _rand((T, Hkv, D), 7)
    o, lse = oracle.fwd(q, k, v, cu, cu, 0.9, True, mutation=mutation)
    off = 0
    for s in lq:
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            ok, msg = _close(o[off, h], v[off, hk], 1e-12)
            if not ok:
                return False, f"causal row 0 O: {msg}"
            ok, msg = _close(lse[h, off], 0.9 * q[off, h] @ k[off, hk], 1e-12)
            if not ok:
                return False, f"causal row 0 LSE: {msg}"
        off += s
    # Q = 0 -> uniform weights over the allowed keys
    qz = np.zeros_like(q)
    for causal in (False, True):
        o, lse = oracle.fwd(qz, k, v, cu, cu, 0.9, causal, mutation=mutation)
        off = 0
        for s in lq:
            for h in range(Hq):
                hk = h // (Hq // Hkv)
                for i in range(s):
                    n = (i + 1) if causal else s
                    ok, msg = _close(o[off + i, h], v[off:off + n, hk].mean(0), 1e-12)
                    if not ok:
                        return False, f"Q=0 causal={causal} O: {msg}"
                    ok, msg = _close(lse[h, off + i], np.log(n), 1e-12)
                    if not ok:
                        return False, f"Q=0 causal={causal} LSE: {msg}"
            off += s
    # a single key: O = v_0 for every query row, LSE = its score
    q1 = _rand((5, 2, D), 8)
    k1 = _rand((1, 1, D), 9)
    v1 = _rand((1, 1, D), 10)
    o, lse = oracle.fwd(q1, k1, v1, _cu([5]), _cu([1]), 0.3, False, mutation=mutation)
    ok, msg = _close(o, np.broadcast_to(v1, o.shape), 1e-12)
    if not ok:
        return False, f"single key O: {msg}"
    ok, msg = _close(lse, 0.3 * np.einsum("thd,d->ht", q1, k1[0, 0]), 1e-12)
    if not ok:
        return False, f"single key LSE: {msg}"
    # shifting every key of a segment by one vector: O unchanged, LSE shifts
    shift = _rand((1, Hkv, D), 11)
    for causal in (False, True):
        o0, l0 = oracle.fwd(q, k, v, cu, cu, 0.9, causal, mutation=mutation)
        o1, l1 = oracle.fwd(q, k + shift, v, cu, cu, 0.9, causal, mutation=mutation)
        ok, msg = _close(o1, o0, 1e-10)
        if not ok:
            return False, f"key shift O causal={causal}: {msg}"
        G = Hq // Hkv
        dl = 0.9 * np.einsum("thd,hd->ht", q, np.repeat(shift[0], G, axis=0))
        ok, msg = _close(l1, l0 + dl, 1e-10)
        if not ok:
            return False, f"key shift LSE causal={causal}: {msg}"
    return True, "ok"


def check_gradient_identities(mutation=0):
    Hq, Hkv, D = 4, 2, 8
    lq = [13, 6]
    cu = _cu(lq)
    T = sum(lq)
    q, k, v, do = (_rand((T, h, D), s) for h, s in ((Hq, 12), (Hkv, 13), (Hkv, 14), (Hq, 15)))
    G = Hq // Hkv
    for causal in (False, True):
        dq, dk, dv = oracle.bwd(q, k, v, do, cu, cu, 0.6, causal, mutation=mutation)
        off = 0
        for s in lq:
            ok, msg = _close(dk[off:off + s].sum(0), np.zeros((Hkv, D)), 1e-12)
            if not ok:
                return False, f"sum dK causal={causal}: {msg}"
            ref = do[off:off + s].sum(0).reshape(Hkv, G, D).sum(1)
            ok, msg = _close(dv[off:off + s].sum(0), ref, 1e-12)
            if not ok:
                return False, f"sum dV causal={causal}: {msg}"
            off += s
    return True, "ok"


def check_structure(mutation=0):
    Hq, Hkv, D = 4, 2, 8
    lq = [5, 9, 1, 7]
    cu = _cu(lq)
    T = sum(lq)
    q, k, v, do = (_rand((T, h, D), s) for h, s in ((Hq, 16), (Hkv, 17), (Hkv, 18), (Hq, 19)))
    G = Hq // Hkv
    for causal in (False, True):
        o, lse = oracle.fwd(q, k, v, cu, cu, 0.4, causal, mutation=mutation)
        dq, dk, dv = oracle.bwd(q, k, v, do, cu, cu, 0.4, causal, mutation=mutation)
        # each segment alone gives bit-identical results
        off = 0
        for s in lq:
            sl = slice(off, off + s)
            c1 = _cu([s])
            o1, l1 = oracle.fwd(q[sl], k[sl], v[sl], c1, c1, 0.4, causal, mutation=mutation)
            d1 = oracle.bwd(q[sl], k[sl], v[sl], do[sl], c1, c1, 0.4, causal, mutation=mutation)
            if not (np.array_equal(o1, o[sl]) and np.array_equal(l1, lse[:, sl])):
                return False, f"varlen segment fwd differs (causal={causal})"
            if not all(np.array_equal(a, b[sl]) for a, b in zip(d1, (dq, dk, dv))):
                return False, f"varlen segment bwd differs (causal={causal})"
            off += s
        # GQA == MHA on K/V repeated per contiguous group
        kr, vr = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)
        om, lm = oracle.fwd(q, kr, vr, cu, cu, 0.4, causal, mutation=mutation)
        dqm, dkm, dvm = oracle.bwd(q, kr, vr, do, cu, cu, 0.4, causal, mutation=mutation)
        for name, a, b in (("O", o, om), ("LSE", lse, lm), ("dQ", dq, dqm),
                           ("dK", dk, dkm.reshape(T, Hkv, G, D).sum(2)),
                           ("dV", dv, dvm.reshape(T, Hkv, G, D).sum(2))):
            ok, msg = _close(a, b, 1e-12)
            if not ok:
                return False, f"GQA vs repeated MHA {name} causal={causal}: {msg}"
    return True, "ok"


def check_rows_match_full(mutation=0):
    Hq, Hkv, D = 4, 1, 8
    lq = [10, 17]
    cu = _cu(lq)
    T = sum(lq)
    q, k, v, do = (_rand((T, h, D), s) for h, s in ((Hq, 20), (Hkv, 21), (Hkv, 22), (Hq, 23)))
    for causal in (False, True):
        o, lse = oracle.fwd(q, k, v, cu, cu, 0.5, causal, mutation=mutation)
        dq, _, _ = oracle.bwd(q, k, v, do, cu, cu, 0.5, causal, mutation=mutation)
        heads = np.array([0, 3, 1, 2, 2], np.int32)
        rows = np.array([0, 9, 10, 26, 13], np.int64)
        ro, rl, rdq = oracle.rows(q, k, v, cu, cu, 0.5, causal, heads, rows, dout=do,
                                  mutation=mutation)
        if not (np.array_equal(ro, o[rows, heads]) and np.array_equal(rl, lse[heads, rows])
                and np.array_equal(rdq, dq[rows, heads])):
            return False, f"sampled rows differ from the full oracle (causal={causal})"
    return True, "ok"


def check_cols_match_full(mutation=0):
    # sampled key rows (dK, dV summed over the group) equal the full backward's,
    # with GQA, two segments, causal both ways, a window and a softcap
    Hq, Hkv, D = 4, 2, 8
    lq = [11, 16]
    cu = _cu(lq)
    T = sum(lq)
    q, k, v, do = (_rand((T, h, D), s) for h, s in ((Hq, 40), (Hkv, 41), (Hkv, 42), (Hq, 43)))
    keys = np.array([0, 10, 11, 26, 17, 3], np.int64)
    khead = np.array([0, 1, 1, 0, 0, 1], np.int32)
    # the last set: only keys near the end of the longer segment, so under a
    # causal mask or a window most rows are never selected for statistics
    tail = (np.array([25, 26, 24, 26], np.int64), np.array([0, 1, 1, 1], np.int32))
    for causal, window, cap, (ks, kh) in ((False, None, 0.0, (keys, khead)),
                                          (True, None, 0.0, (keys, khead)),
                                          (True, (4, 0), 0.0, (keys, khead)),
                                          (False, None, 2.5, (keys, khead)),
                                          (True, None, 0.0, tail),
                                          (False, (2, 1), 0.0, tail)):
        _, dk, dv = oracle.bwd(q, k, v, do, cu, cu, 0.5, causal, window=window, softcap=cap,
                               mutation=mutation)
        cdk, cdv = oracle.cols(q, k, v, do, cu, cu, 0.5, causal, kh, ks, window=window,
                               softcap=cap, mutation=mutation)
        if not (np.array_equal(cdk, dk[ks, kh]) and np.array_equal(cdv, dv[ks, kh])):
            return False, (f"sampled key rows differ from the full oracle "
                           f"(causal={causal}, window={window}, softcap={cap}, keys={list(ks)})")
    return True, "ok"


def check_fully_masked_rows(mutation=0):
    # causal with s_q > s_k: the first s_q - s_k rows see no key at all
    q = _rand((6, 1, 4), 24)
    k = _rand((3, 1, 4), 25)
    v = _rand((3, 1, 4), 26)
    do = _rand((6, 1, 4), 27)
    o, lse = oracle.fwd(q, k, v, _cu([6]), _cu([3]), 1.0, True, mutation=mutation)
    if not (np.all(o[:3] == 0) and np.all(np.isneginf(lse[0, :3])) and np.all(np.isfinite(lse[0, 3:]))):
        return False, "fully masked rows are not O=0, LSE=-inf"
    dq, dk, dv = oracle.bwd(q, k, v, do, _cu([6]), _cu([3]), 1.0, True, mutation=mutation)
    if not (np.all(dq[:3] == 0) and np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))):
        return False, "fully masked rows leak into gradients"
    return True, "ok"


# --------------------------------------------------------------------------
# local (sliding-window) masks and the softcap
# --------------------------------------------------------------------------
def check_window_softcap_closed_forms(mutation=0):
    Hq, Hkv, D = 2, 1, 8
    lq, lk = [7, 5], [9, 5]          # s_k - s_q = 2 and 0
    cq, ck = _cu(lq), _cu(lk)
    q, k, v = _rand((12, Hq, D), 90), _rand((14, Hkv, D), 91), _rand((14, Hkv, D), 92)
    scale = 0.6
    # window (0, 0): row i sees exactly key i + (s_k - s_q): O = v_j, LSE = s_ij
    for cap in (0.0, 2.5):
        o, lse = oracle.fwd(q, k, v, cq, ck, scale, False, window=(0, 0), softcap=cap,
                            mutation=mutation)
        oq = ok_ = 0
        for sq, sk in zip(lq, lk):
            for i in range(sq):
                j = i + sk - sq
                for h in range(Hq):
                    a = scale * float(q[oq + i, h] @ k[ok_ + j, 0])
                    want = cap * np.tanh(a / cap) if cap > 0 else a
                    if not np.allclose(o[oq + i, h], v[ok_ + j, 0], atol=1e-14):
                        return False, f"window (0,0) cap={cap}: O is not v_(i+delta)"
                    if abs(lse[h, oq + i] - want) > 1e-12:
                        return False, f"window (0,0) cap={cap}: LSE {lse[h, oq + i]} vs {want}"
            oq += sq
            ok_ += sk
    # bounds at least as wide as the segment change nothing; (-1, 0) is causal
    o0, l0 = oracle.fwd(q, k, v, cq, ck, scale, False, mutation=mutation)
    o1, l1 = oracle.fwd(q, k, v, cq, ck, scale, False, window=(20, 20), mutation=mutation)
    if not (_close(o1, o0, 1e-14)[0] and _close(l1, l0, 1e-14)[0]):
        return False, "a window wider than the segment changed the result"
    oc_, lc = oracle.fwd(q, k, v, cq, ck, scale, True, mutation=mutation)
    ow, lw = oracle.fwd(q, k, v, cq, ck, scale, False, window=(-1, 0), mutation=mutation)
    if not (_close(ow, oc_, 1e-14)[0] and _close(lw, lc, 1e-14)[0]):
        return False, "window (-1, 0) differs from causal"
    # a huge cap is no cap (tanh(x) = x to O(x^3))
    oh, lh = oracle.fwd(q, k, v, cq, ck, scale, False, softcap=1e7, mutation=mutation)
    if not (_close(oh, o0, 1e-9)[0] and _close(lh, l0, 1e-9)[0]):
        return False, "softcap 1e7 differs from no softcap"
    return True, "ok"


def check_window_is_a_slice(mutation=0):
    """Row i under window (L, R) equals unmasked attention over the key slice
    [i + delta - L, i + delta + R] (clipped to the segment), computed by the
    unmasked oracle on that slice alone."""
    Hq, Hkv, D = 2, 2, 4
    sq, sk = 9, 12
    q, k, v = _rand((sq, Hq, D), 93), _rand((sk, Hkv, D), 94), _rand((sk, Hkv, D), 95)
    for (L, R) in ((2, 1), (0, 3), (4, 0), (3, -1), (-1, 2)):
        o, lse = oracle.fwd(q, k, v, _cu([sq]), _cu([sk]), 0.8, False, window=(L, R),
                            mutation=mutation)
        for i in range(sq):
            d = i + sk - sq
            lo = 0 if L < 0 else max(0, d - L)
            hi = sk - 1 if R < 0 else min(sk - 1, d + R)
            if hi < lo:
                if not (np.all(o[i] == 0) and np.all(np.isneginf(lse[:, i]))):
                    return False, f"window {(L, R)} row {i}: empty window not O=0, LSE=-inf"
                continue
            os_, ls_ = oracle.fwd(q[i:i + 1], k[lo:hi + 1], v[lo:hi + 1], _cu([1]),
                                  _cu([hi + 1 - lo]), 0.8, False, mutation=mutation)
            if not (_close(o[i:i + 1], os_, 1e-13)[0] and _close(lse[:, i:i + 1], ls_, 1e-13)[0]):
                return False, f"window {(L, R)} row {i} differs from its key slice"
    return True, "ok"


MASK_CASES = [
    # (lengths_q, lengths_k, Hq, Hkv, D, causal, window, softcap)
    ([7], [7], 2, 1, 4, False, (2, 1), 0.0),
    ([6, 4], [8, 4], 2, 1, 4, True, (3, -1), 0.0),
    ([7], [7], 2, 2, 4, False, (-1, -1), 1.5),
    ([5, 6], [5, 7], 4, 2, 4, True, (2, 0), 2.0),
]


def check_torch_reference_masks(mutation=0, tol=1e-12):
    for ci, (lq, lk, Hq, Hkv, D, causal, win, cap) in enumerate(MASK_CASES):
        Tq, Tk = sum(lq), sum(lk)
        q, k, v = _rand((Tq, Hq, D), 150 + ci), _rand((Tk, Hkv, D), 160 + ci), _rand((Tk, Hkv, D), 170 + ci)
        do = _rand((Tq, Hq, D), 180 + ci)
        scale = 0.9
        cq, ck = _cu(lq), _cu(lk)
        o, lse = oracle.fwd(q, k, v, cq, ck, scale, causal, window=win, softcap=cap,
                            mutation=mutation)
        dq, dk, dv = oracle.bwd(q, k, v, do, cq, ck, scale, causal, window=win, softcap=cap,
                                mutation=mutation)
        ro, rlse, (rdq, rdk, rdv) = torch_reference(q, k, v, do, lq, lk, scale, causal,
                                                    window=win, softcap=cap)
        for name, a, b in (("O", o, ro), ("LSE", lse, rlse), ("dQ", dq, rdq),
                           ("dK", dk, rdk), ("dV", dv, rdv)):
            ok, msg = _close(a, b, tol)
            if not ok:
                return False, f"torch mask case {ci} {name}: {msg}"
    return True, "ok"


def check_finite_differences_masks(mutation=0, eps=1e-6, tol=1e-6):
    for ci, (lq, lk, Hq, Hkv, D, causal, win, cap) in enumerate(MASK_CASES):
        Tq, Tk = sum(lq), sum(lk)
        q, k, v = _rand((Tq, Hq, D), 110 + ci), _rand((Tk, Hkv, D), 120 + ci), _rand((Tk, Hkv, D), 130 + ci)
        do = _rand((Tq, Hq, D), 140 + ci)
        scale = 0.7
        cq, ck = _cu(lq), _cu(lk)
        dq, dk, dv = oracle.bwd(q, k, v, do, cq, ck, scale, causal, window=win, softcap=cap,
                                mutation=mutation)

        def loss():
            o, _ = oracle.fwd(q, k, v, cq, ck, scale, causal, window=win, softcap=cap,
                              mutation=mutation)
            return float(np.sum(o * do))

        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            flat = x.reshape(-1)
            for t in range(flat.size):
                old = flat[t]
                flat[t] = old + eps
                lp = loss()
                flat[t] = old - eps
                lm = loss()
                flat[t] = old
                num.reshape(-1)[t] = (lp - lm) / (2 * eps)
            ok, msg = _close(g, num, tol)
            if not ok:
                return False, f"FD mask case {ci} d{name}: {msg}"
    return True, "ok"


ALL_CHECKS = [
    check_window_softcap_closed_forms,
    check_window_is_a_slice,
    check_closed_forms,
    check_lse_logsumexp,
    check_gradient_identities,
    check_structure,
    check_rows_match_full,
    check_cols_match_full,
    check_fully_masked_rows,
    check_torch_reference,
    check_torch_reference_masks,
    check_finite_differences,
    check_finite_differences_masks,
]
