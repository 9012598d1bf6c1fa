"""fp64 CPU oracle for exact scaled-dot-product attention -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does, and this
package never imports the CUDA library: the two share no code.  The only thing
both sides use is the seeded input generator, which holds none of the method's
arithmetic.

The arithmetic lives in ``attn_oracle.c`` (plain C, double precision, OpenMP
over independent rows); this module compiles it with gcc on first use and
marshals numpy arrays through ctypes.  Layouts follow the library: q/out/dout/dq
``[Tq, Hq, D]``, k/v/dk/dv ``[Tk, Hkv, D]``, lse ``[Hq, Tq]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LOCK = threading.Lock()
_LIBS: dict = {}


def lib_path(mutation: int = 0, out_dir: str | None = None) -> str:
    name = "liboracle.so" if mutation == 0 else f"liboracle_mut{mutation}.so"
    return os.path.join(out_dir or _HERE, name)


def build(mutation: int = 0, out_dir: str | None = None, force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math).

    ``mutation`` > 0 builds a copy with one planted mistake; the suite uses
    those copies to show its pins catch such mistakes.
    """
    path = lib_path(mutation, out_dir)
    if force or not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
        tmp = path + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", f"-DORACLE_MUTATION={int(mutation)}", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, path)
    return path


def _load(mutation: int = 0, out_dir: str | None = None):
    key = (mutation, out_dir)
    with _LOCK:
        if key not in _LIBS:
            lib = ctypes.CDLL(build(mutation, out_dir))
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            lp = ctypes.POINTER(ctypes.c_int64)
            i, d = ctypes.c_int, ctypes.c_double
            lg = ctypes.c_long
            lib.oracle_fwd.argtypes = [dp, dp, dp, ip, ip, i, i, i, i, d, i, dp, dp]
            lib.oracle_bwd.argtypes = [dp, dp, dp, dp, ip, ip, i, i, i, i, d, i, dp, dp, dp]
            lib.oracle_rows.argtypes = [dp, dp, dp, dp, ip, ip, i, i, i, i, d, i, i, ip, lp,
                                        dp, dp, dp]
            lib.oracle_fwd_ex.argtypes = [dp, dp, dp, ip, ip, i, i, i, i, d, i, lg, lg, d, dp,
                                          dp]
            lib.oracle_bwd_ex.argtypes = [dp, dp, dp, dp, ip, ip, i, i, i, i, d, i, lg, lg, d,
                                          dp, dp, dp]
            lib.oracle_rows_ex.argtypes = [dp, dp, dp, dp, ip, ip, i, i, i, i, d, i, lg, lg, d,
                                           i, ip, lp, dp, dp, dp]
            lib.oracle_cols_ex.argtypes = [dp, dp, dp, dp, ip, ip, i, i, i, i, d, i, lg, lg, d,
                                           i, ip, lp, dp, dp]
            for fn in (lib.oracle_fwd, lib.oracle_bwd, lib.oracle_rows, lib.oracle_fwd_ex,
                       lib.oracle_bwd_ex, lib.oracle_rows_ex, lib.oracle_cols_ex):
                fn.restype = ctypes.c_int
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_mutation.restype = ctypes.c_int
            _LIBS[key] = lib
        return _LIBS[key]


def _f64(x) -> np.ndarray:
    """Any array-like (numpy, torch CPU of any float dtype) -> contiguous float64."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: only needed for torch inputs

        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _dims(q, k, cu_q):
    Tq, Hq, D = q.shape
    Tk, Hkv, Dk = k.shape
    assert Dk == D, "q and k head_dim differ"
    return Tq, Hq, Tk, Hkv, D, len(cu_q) - 1


def num_threads(mutation: int = 0) -> int:
    return int(_load(mutation).oracle_num_threads())


def _mask_args(window, softcap):
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    return wl, wr, float(softcap or 0.0)


def fwd(q, k, v, cu_q, cu_k, scale, causal, *, window=None, softcap=0.0, mutation: int = 0,
        lib_dir=None):
    """O [Tq,Hq,D] and LSE [Hq,Tq] (natural log of the scaled scores), float64.

    ``window`` = (left, right) key-distance bounds around the bottom-right
    aligned diagonal (negative = no bound); ``softcap`` > 0 caps the scaled
    scores at c * tanh(s / c)."""
    wl, wr, cap = _mask_args(window, softcap)
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu_q, cu_k = _i32(cu_q), _i32(cu_k)
    Tq, Hq, Tk, Hkv, D, B = _dims(q, k, cu_q)
    assert int(cu_q[-1]) == Tq and int(cu_k[-1]) == Tk
    out = np.zeros((Tq, Hq, D), np.float64)
    lse = np.zeros((Hq, Tq), np.float64)
    rc = _load(mutation, lib_dir).oracle_fwd_ex(
        _ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
        _ptr(cu_q, ctypes.c_int32), _ptr(cu_k, ctypes.c_int32), B, Hq, Hkv, D,
        float(scale), int(bool(causal)), wl, wr, cap, _ptr(out, ctypes.c_double),
        _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_fwd rejected its arguments (code {rc})")
    return out, lse


def bwd(q, k, v, dout, cu_q, cu_k, scale, causal, *, window=None, softcap=0.0,
        mutation: int = 0, lib_dir=None):
    """dQ [Tq,Hq,D], dK, dV [Tk,Hkv,D] of L = sum(dout * O), float64."""
    wl, wr, cap = _mask_args(window, softcap)
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    cu_q, cu_k = _i32(cu_q), _i32(cu_k)
    Tq, Hq, Tk, Hkv, D, B = _dims(q, k, cu_q)
    assert dout.shape == q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rc = _load(mutation, lib_dir).oracle_bwd_ex(
        _ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
        _ptr(dout, ctypes.c_double), _ptr(cu_q, ctypes.c_int32), _ptr(cu_k, ctypes.c_int32),
        B, Hq, Hkv, D, float(scale), int(bool(causal)), wl, wr, cap, _ptr(dq, ctypes.c_double),
        _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_bwd rejected its arguments (code {rc})")
    return dq, dk, dv


def rows(q, k, v, cu_q, cu_k, scale, causal, heads, row_index, dout=None, *,
         window=None, softcap=0.0, mutation: int = 0, lib_dir=None):
    """O, LSE (and dQ if ``dout`` is given) for chosen (head, global row) pairs.

    Exact at any length: a row needs only its own scores.  Returns
    ``(out [n,D], lse [n], dq [n,D] or None)``.
    """
    wl, wr, cap = _mask_args(window, softcap)
    q, k, v = _f64(q), _f64(k), _f64(v)
    dptr = None
    if dout is not None:
        dout = _f64(dout)
        dptr = _ptr(dout, ctypes.c_double)
    cu_q, cu_k = _i32(cu_q), _i32(cu_k)
    Tq, Hq, Tk, Hkv, D, B = _dims(q, k, cu_q)
    heads = _i32(heads)
    row_index = np.ascontiguousarray(np.asarray(row_index, dtype=np.int64))
    n = len(heads)
    assert len(row_index) == n
    out = np.zeros((n, D), np.float64)
    lse = np.zeros((n,), np.float64)
    dq = np.zeros((n, D), np.float64) if dout is not None else None
    rc = _load(mutation, lib_dir).oracle_rows_ex(
        _ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double), dptr,
        _ptr(cu_q, ctypes.c_int32), _ptr(cu_k, ctypes.c_int32), B, Hq, Hkv, D, float(scale),
        int(bool(causal)), wl, wr, cap, n, _ptr(heads, ctypes.c_int32),
        _ptr(row_index, ctypes.c_int64),
        _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double),
        _ptr(dq, ctypes.c_double) if dq is not None else None)
    if rc != 0:
        raise ValueError(f"oracle_rows rejected its arguments (code {rc})")
    return out, lse, dq


def cols(q, k, v, dout, cu_q, cu_k, scale, causal, kv_heads, key_index, *,
         window=None, softcap=0.0, mutation: int = 0, lib_dir=None):
    """dK and dV for chosen (kv head, global key row) pairs, summed over the
    query heads of the group.

    Exact at any length; a key row needs every query row's LSE and D_i, so the
    forward statistics of the segments and heads involved are computed first
    (their full forward).  Returns ``(dk [n,D], dv [n,D])``.
    """
    wl, wr, cap = _mask_args(window, softcap)
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    cu_q, cu_k = _i32(cu_q), _i32(cu_k)
    Tq, Hq, Tk, Hkv, D, B = _dims(q, k, cu_q)
    kv_heads = _i32(kv_heads)
    key_index = np.ascontiguousarray(np.asarray(key_index, dtype=np.int64))
    n = len(kv_heads)
    assert len(key_index) == n
    dk = np.zeros((n, D), np.float64)
    dv = np.zeros((n, D), np.float64)
    rc = _load(mutation, lib_dir).oracle_cols_ex(
        _ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
        _ptr(dout, ctypes.c_double), _ptr(cu_q, ctypes.c_int32), _ptr(cu_k, ctypes.c_int32),
        B, Hq, Hkv, D, float(scale), int(bool(causal)), wl, wr, cap, n,
        _ptr(kv_heads, ctypes.c_int32), _ptr(key_index, ctypes.c_int64),
        _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_cols rejected its arguments (code {rc})")
    return dk, dv
