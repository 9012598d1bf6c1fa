"""Ahead-of-time build of libattn.so (sm_100a) with nvcc, in the source tree.

Usage: python -m exact_attention_129_b200.build [--force] [--debug]
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libattn.so")
SOURCES = ["api.cu"]
HEADERS = ["ptx.cuh", "fwd_kernel.cuh", "fwd_pair_kernel.cuh", "bwd_kernels.cuh",
           "bwd_pair_kernel.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "attn.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs() if os.path.exists(f))


def build(force: bool = False, verbose: bool = False, extra=(), out: str | None = None) -> str:
    """Compile libattn.so (or, with ``out``, a variant with the extra nvcc
    arguments ``extra``, e.g. ``-DATTN_FWD_POLY_PAIRS=2``, at that path)."""
    target = out or LIB
    if out is None and not force and up_to_date():
        return LIB
    tmp = target + f".tmp{os.getpid()}"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
           "--expt-relaxed-constexpr", "-Xptxas", "-v" if verbose else "-O3",
           *extra, *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libattn.so")
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
