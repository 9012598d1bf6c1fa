"""CPU tests: the fp64 oracle against its pins (nothing here needs a GPU)."""
import json
import os
import tempfile

import numpy as np
import pytest

import oracle
from tests import oracle_checks as oc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_key_closed_form.json")


@pytest.mark.parametrize("check", oc.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    ok, msg = check()
    assert ok, msg


def test_golden_two_key_closed_form():
    g = json.load(open(GOLDEN))
    nc = g["non_causal"]
    q, k, v, do = (np.array(nc[x]) for x in ("q", "k", "v", "dout"))
    cq, ck = np.array([0, 1], np.int32), np.array([0, 2], np.int32)
    o, lse = oracle.fwd(q, k, v, cq, ck, 1.0, False)
    np.testing.assert_allclose(o, nc["out"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, nc["lse"], rtol=0, atol=1e-14)
    dq, dk, dv = oracle.bwd(q, k, v, do, cq, ck, 1.0, False)
    np.testing.assert_allclose(dq, nc["dq"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk, nc["dk"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv, nc["dv"], rtol=0, atol=1e-14)
    c = g["causal"]
    cu = np.array([0, 2], np.int32)
    o, lse = oracle.fwd(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]), cu, cu, 1.0, True)
    np.testing.assert_allclose(o, c["out"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, c["lse"], rtol=0, atol=1e-14)


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(0)
    lq = [37, 64, 5]
    cu = np.zeros(4, np.int32)
    cu[1:] = np.cumsum(lq)
    T = sum(lq)
    q, k, v, do = (rng.standard_normal((T, h, 16)) for h in (4, 2, 2, 4))
    ref = oracle.fwd(q, k, v, cu, cu, 0.25, True) + oracle.bwd(q, k, v, do, cu, cu, 0.25, True)
    old = os.environ.get("OMP_NUM_THREADS")
    # a separate process picks up a different thread count
    import subprocess
    import sys
    code = (
        "import numpy as np, oracle, sys; "
        "rng=np.random.default_rng(0); lq=[37,64,5]; cu=np.zeros(4,np.int32); cu[1:]=np.cumsum(lq); T=sum(lq); "
        "q,k,v,do=(rng.standard_normal((T,h,16)) for h in (4,2,2,4)); "
        "r=oracle.fwd(q,k,v,cu,cu,0.25,True)+oracle.bwd(q,k,v,do,cu,cu,0.25,True); "
        "np.savez(sys.argv[1], *r)")
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "r.npz")
        env = dict(os.environ, OMP_NUM_THREADS="1",
                   PYTHONPATH=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        subprocess.run([sys.executable, "-c", code, path], check=True, env=env)
        got = np.load(path)
        for i, a in enumerate(ref):
            assert np.array_equal(got[f"arr_{i}"], a)
    assert old == os.environ.get("OMP_NUM_THREADS")


def test_rejects_bad_arguments():
    q = np.zeros((4, 3, 8))
    k = np.zeros((4, 2, 8))
    cu = np.array([0, 4], np.int32)
    with pytest.raises(ValueError):
        oracle.fwd(q, k, k, cu, cu, 1.0, False)  # 3 q heads not a multiple of 2 kv heads
    with pytest.raises(ValueError):
        oracle.fwd(np.zeros((4, 2, 8)), k, k, np.array([1, 4], np.int32), cu, 1.0, False)


MUTATIONS = {
    1: "dQ loses its scale factor",
    2: "dS has its sign flipped",
    3: "causal mask drops the diagonal",
    4: "GQA maps heads interleaved instead of in contiguous groups",
    5: "LSE drops the max term",
    6: "dK multiplies dS by dO instead of Q",
    7: "D_i drops the O factor",
    8: "the window's far edge is excluded",
    9: "the softcap's derivative is dropped from dS",
    10: "the softcap is applied to the unscaled score",
    11: "the sampled-key oracle leaves the diagonal row out of its selection",
}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS), ids=lambda m: MUTATIONS[m])
def test_pins_catch_planted_mistake(mutation, tmp_path_factory):
    """Each planted mistake in a copy of the oracle fails at least one pin."""
    d = str(tmp_path_factory.mktemp(f"mut{mutation}"))
    oracle.build(mutation, out_dir=d)
    caught = []
    for check in oc.ALL_CHECKS:
        if check is oc.check_finite_differences and caught:
            break  # the slowest check is only needed if nothing cheaper failed
        ok, msg = check_in(check, mutation, d)
        if not ok:
            caught.append(f"{check.__name__}: {msg}")
    assert caught, f"no pin caught mutation {mutation} ({MUTATIONS[mutation]})"


def check_in(check, mutation, lib_dir):
    # route every oracle call of the check to the mutant library in lib_dir
    orig = (oracle.fwd, oracle.bwd, oracle.rows, oracle.cols)
    oracle.fwd = lambda *a, **kw: orig[0](*a, **{**kw, "lib_dir": lib_dir})
    oracle.bwd = lambda *a, **kw: orig[1](*a, **{**kw, "lib_dir": lib_dir})
    oracle.rows = lambda *a, **kw: orig[2](*a, **{**kw, "lib_dir": lib_dir})
    oracle.cols = lambda *a, **kw: orig[3](*a, **{**kw, "lib_dir": lib_dir})
    try:
        return check(mutation=mutation)
    finally:
        oracle.fwd, oracle.bwd, oracle.rows, oracle.cols = orig
