"""GPU parity of the forward built with its FMA-pipe exp2.

The forward softmax can take a fraction of its 2^x on the FMA pipe, with a
degree-3 polynomial after range reduction (exp2_fma_pair in ptx.cuh, constants
from exp2_poly_fit.py, checked on the CPU in test_exp2_poly.py), instead of on
the special-function unit; ATTN_FWD_POLY_PAIRS of every 8 score pairs of
unmasked blocks do so.  The default build sets it to 0 (no variant measured
faster).  Here the variants with 2 and 4 are built into a temporary directory
and the head_dim-128 forward parity tests (and two full-size workloads) run
against the oracle with that library loaded, in a child process.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SELECT = ("128 and (ragged or gqa8 or sq_ne_sk or epilogue or pack_gqa_forced or lse_flag "
          "or large_scores or deterministic)")


@pytest.mark.parametrize("pairs", [2, 4])
def test_forward_with_fma_exp2(pairs, tmp_path):
    from exact_attention_129_b200 import build

    lib = build.build(out=str(tmp_path / f"libattn_poly{pairs}.so"),
                      extra=[f"-DATTN_FWD_POLY_PAIRS={pairs}"])
    env = dict(os.environ, ATTN_LIBRARY=lib)
    probe = "import exact_attention_129_b200 as ea; print(ea.library().attn_version().decode())"
    ver = subprocess.run([sys.executable, "-c", probe], env=env, cwd=ROOT, capture_output=True,
                         text=True, check=True).stdout
    assert f"fwd_poly_pairs={pairs}" in ver, ver
    base = [sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu"]
    for args in (["tests/test_fwd_gpu.py", "-k", SELECT],
                 ["tests/test_full_size_gpu.py", "-k", "varlen_gqa or gqa_16k"]):
        r = subprocess.run(base + args, env=env, cwd=ROOT, capture_output=True, text=True)
        assert r.returncode == 0, (r.stdout[-4000:] + r.stderr[-2000:])
        assert " passed" in r.stdout and " failed" not in r.stdout, r.stdout[-2000:]
