"""Exact attention on B200 (sm_100a): thin Python binding over libattn.so.

Every step of the computation runs in the CUDA kernels behind the C ABI in
``include/attn.h``; this module only marshals torch tensors (device memory,
current stream) into that ABI.  There is no CPU fallback: if the library is
missing or the tensors are not on a CUDA device, calls raise.

Functions
---------
attn_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, ...)
    -> (out, lse); causal, window=(left, right) and softcap options
attn_bwd(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, ...)
    -> (dq, dk, dv)
attention(...)  autograd-aware forward (backward through attn_bwd)
last_device_error() -> (status, message)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["attn_fwd", "attn_bwd", "attention", "bwd_workspace_size", "fwd_split_workspace_size",
           "last_device_error",
           "set_timing_events", "KERNEL_FWD", "KERNEL_BWD_MAIN",
           "library", "LIB_PATH", "AttnError", "STATUS"]

# ATTN_LIBRARY names another build of the same library (a variant built with
# exact_attention_129_b200.build.build(out=..., extra=...)); default: the in-tree build
LIB_PATH = os.environ.get("ATTN_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libattn.so")
STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED",
          3: "ATTN_ERR_CUDA", 4: "ATTN_ERR_TIMEOUT", 5: "ATTN_ERR_SCRATCH_TOO_SMALL"}
EXPORTED = ("attn_fwd", "attn_bwd", "attn_fwd_ex", "attn_bwd_ex", "attn_fwd_split",
            "attn_fwd_split_workspace_size", "attn_bwd_workspace_size",
            "attn_last_device_error", "attn_set_timing_events", "attn_bwd_static_scratch",
            "attn_watchdog_selftest", "attn_version")
KERNEL_FWD, KERNEL_BWD_MAIN = 0, 1


class AttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


_lib = None


def library() -> ctypes.CDLL:
    """Load libattn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m exact_attention_129_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
        lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                 f32, i32, i32, vp, vp, vp]
        lib.attn_fwd.restype = ctypes.c_int
        lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                 i32, i32, f32, i32, vp, vp, vp, vp, ctypes.c_size_t, vp]
        lib.attn_bwd.restype = ctypes.c_int
        lib.attn_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                    i32, f32, i32, i32, i32, f32, i32, vp, vp, vp]
        lib.attn_fwd_ex.restype = ctypes.c_int
        lib.attn_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                    i32, i32, i32, f32, i32, i32, i32, f32, vp, vp, vp, vp,
                                    ctypes.c_size_t, vp]
        lib.attn_bwd_ex.restype = ctypes.c_int
        lib.attn_fwd_split.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                       i32, f32, i32, i32, i32, f32, i32, i32, vp, vp, vp,
                                       ctypes.c_size_t, vp]
        lib.attn_fwd_split.restype = ctypes.c_int
        lib.attn_fwd_split_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.attn_fwd_split_workspace_size.restype = ctypes.c_size_t
        lib.attn_bwd_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.attn_bwd_workspace_size.restype = ctypes.c_size_t
        lib.attn_last_device_error.argtypes = [vp, ctypes.c_char_p, ctypes.c_size_t]
        lib.attn_last_device_error.restype = ctypes.c_int
        lib.attn_version.restype = ctypes.c_char_p
        lib.attn_set_timing_events.argtypes = [i32, vp, vp]
        lib.attn_set_timing_events.restype = ctypes.c_int
        lib.attn_bwd_static_scratch.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                                i32, i32, i32, i32, i32, f32, i32, vp, vp, vp,
                                                vp]
        lib.attn_bwd_static_scratch.restype = ctypes.c_int
        lib.attn_watchdog_selftest.argtypes = [i32, vp]
        lib.attn_watchdog_selftest.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("exact_attention_129_b200 runs on CUDA tensors only")


def _check_layout(name, t, dtype):
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_like(name, t, shape, dtype, dev):
    """A caller-supplied buffer must match what the kernels will read or write:
    the C ABI takes raw pointers, so a smaller tensor would be overrun."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    _check_layout(name, t, dtype)
    if t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")


def _check_problem(q, k, v, cu_seqlens_q, cu_seqlens_k):
    """Shapes, dtypes and devices of one attention problem (before any launch)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        if t.dim() != 3:
            raise ValueError(f"{n} must be [tokens, heads, head_dim], got shape {tuple(t.shape)}")
        _check_layout(n, t, torch.bfloat16)
    if tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"v must have the shape of k {tuple(k.shape)}, got {tuple(v.shape)}")
    if k.shape[2] != q.shape[2]:
        raise ValueError(f"q and k head_dim differ: {q.shape[2]} and {k.shape[2]}")
    if k.shape[1] < 1 or q.shape[1] % k.shape[1] != 0:
        raise ValueError(f"nheads_q {q.shape[1]} is not a multiple of nheads_kv {k.shape[1]}")
    for n, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if t.dim() != 1 or t.numel() < 2:
            raise ValueError(f"{n} must be a 1-D int32 tensor of batch + 1 offsets")
        _check_layout(n, t, torch.int32)
    if cu_seqlens_q.numel() != cu_seqlens_k.numel():
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length")
    for n, t in (("k", k), ("v", v), ("cu_seqlens_q", cu_seqlens_q),
                 ("cu_seqlens_k", cu_seqlens_k)):
        if t.device != q.device:
            raise ValueError(f"{n} is on {t.device}, q on {q.device}")


def _window(window):
    if window is None:
        return -1, -1
    left, right = window
    return (-1 if left is None else int(left)), (-1 if right is None else int(right))


def fwd_split_workspace_size(total_q, nheads_q, head_dim, num_splits) -> int:
    return int(library().attn_fwd_split_workspace_size(total_q, nheads_q, head_dim, num_splits))


def attn_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, *,
             scale=None, causal=False, window=None, softcap=0.0, return_lse=True, out=None,
             lse=None, num_splits=1, workspace=None):
    """Forward pass. q [Tq,Hq,D], k/v [Tk,Hkv,D] bf16; returns (out, lse or None).

    ``window`` = (left, right): with delta = s_k - s_q, row i sees keys
    [i + delta - left, i + delta + right]; None or a negative side = no bound.
    ``softcap`` > 0 caps each scaled score at softcap * tanh(s / softcap).
    ``num_splits`` > 1 runs the SplitKV forward (key range of every query tile
    cut into that many parts, merged by LSE) in ``workspace`` (allocated if None)."""
    _check_problem(q, k, v, cu_seqlens_q, cu_seqlens_k)
    tq, hq, d = q.shape
    tk, hkv, _ = k.shape
    _check_like("out", out, q.shape, torch.bfloat16, q.device)
    _check_like("lse", lse, (hq, tq), torch.float32, q.device)
    _check_cuda(q, k, v, cu_seqlens_q, cu_seqlens_k, out, lse)
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((hq, tq), device=q.device, dtype=torch.float32)
    wl, wr = _window(window)
    if int(num_splits) > 1:
        need = fwd_split_workspace_size(tq, hq, d, int(num_splits))
        if workspace is None:
            workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
        _check_cuda(workspace)
        if not workspace.is_contiguous() or workspace.device != q.device:
            raise ValueError("workspace must be a contiguous tensor on q's device")
        rc = library().attn_fwd_split(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
            cu_seqlens_q.numel() - 1, tq, tk, int(max_seqlen_q), int(max_seqlen_k), hq, hkv, d,
            float(scale), int(bool(causal)), wl, wr, float(softcap or 0.0), int(num_splits),
            int(bool(return_lse)), _ptr(out), _ptr(lse) if return_lse else None,
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(q.device))
        if rc != 0:
            raise AttnError("attn_fwd_split", rc)
        return out, (lse if return_lse else None)
    rc = library().attn_fwd_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
        cu_seqlens_q.numel() - 1, tq, tk, int(max_seqlen_q), int(max_seqlen_k), hq, hkv, d,
        float(scale), int(bool(causal)), wl, wr, float(softcap or 0.0),
        int(bool(return_lse)), _ptr(out), _ptr(lse) if return_lse else None, _stream(q.device))
    if rc != 0:
        raise AttnError("attn_fwd", rc)
    return out, (lse if return_lse else None)


def bwd_workspace_size(batch, total_q, nheads_q, head_dim) -> int:
    return int(library().attn_bwd_workspace_size(batch, total_q, nheads_q, head_dim))


def attn_bwd(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
             *, scale=None, causal=False, window=None, softcap=0.0, dq=None, dk=None, dv=None,
             workspace=None):
    """Backward pass; returns (dq, dk, dv) in the layouts of q, k, v.  ``causal``,
    ``window`` and ``softcap`` must match the forward call."""
    _check_problem(q, k, v, cu_seqlens_q, cu_seqlens_k)
    tq, hq, d = q.shape
    tk, hkv, _ = k.shape
    if out is None or lse is None or dout is None:
        raise ValueError("out, lse and dout are required")
    _check_like("out", out, q.shape, torch.bfloat16, q.device)
    _check_like("dout", dout, q.shape, torch.bfloat16, q.device)
    _check_like("lse", lse, (hq, tq), torch.float32, q.device)
    _check_like("dq", dq, q.shape, torch.bfloat16, q.device)
    _check_like("dk", dk, k.shape, torch.bfloat16, q.device)
    _check_like("dv", dv, v.shape, torch.bfloat16, q.device)
    if workspace is not None and (not workspace.is_contiguous() or workspace.device != q.device):
        raise ValueError("workspace must be a contiguous tensor on q's device")
    _check_cuda(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, dq, dk, dv, workspace)
    batch = cu_seqlens_q.numel() - 1
    if scale is None:
        scale = d ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_size(batch, tq, hq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    wl, wr = _window(window)
    rc = library().attn_bwd_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(cu_seqlens_q),
        _ptr(cu_seqlens_k), batch, tq, tk, int(max_seqlen_q), int(max_seqlen_k), hq, hkv, d,
        float(scale), int(bool(causal)), wl, wr, float(softcap or 0.0), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(q.device))
    if rc != 0:
        raise AttnError("attn_bwd", rc)
    return dq, dk, dv


def set_timing_events(kernel: int, start=None, stop=None):
    """Record torch.cuda.Event pair around one kernel of later calls (None: off)."""
    if start is not None and (start.cuda_event == 0 or stop.cuda_event == 0):
        raise ValueError("record the events once before passing them (torch creates them lazily)")
    sp = ctypes.c_void_p(start.cuda_event) if start is not None else None
    ep = ctypes.c_void_p(stop.cuda_event) if stop is not None else None
    rc = library().attn_set_timing_events(int(kernel), sp, ep)
    if rc != 0:
        raise AttnError("attn_set_timing_events", rc)


def last_device_error(stream=None):
    """Synchronise the stream and read/clear the device error word."""
    buf = ctypes.create_string_buffer(256)
    s = ctypes.c_void_p(stream.cuda_stream) if stream is not None else \
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = library().attn_last_device_error(s, buf, 256)
    return rc, buf.value.decode()


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, cu_q, cu_k, max_q, max_k, scale, causal, window, softcap):
        out, lse = attn_fwd(q, k, v, cu_q, cu_k, max_q, max_k, scale=scale, causal=causal,
                            window=window, softcap=softcap, return_lse=True)
        ctx.save_for_backward(q, k, v, out, lse, cu_q, cu_k)
        ctx.args = (max_q, max_k, scale, causal, window, softcap)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse, cu_q, cu_k = ctx.saved_tensors
        max_q, max_k, scale, causal, window, softcap = ctx.args
        dq, dk, dv = attn_bwd(q, k, v, out, lse, dout.contiguous(), cu_q, cu_k, max_q, max_k,
                              scale=scale, causal=causal, window=window, softcap=softcap)
        return dq, dk, dv, None, None, None, None, None, None, None, None


def attention(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, *,
              scale=None, causal=False, window=None, softcap=0.0):
    """Differentiable exact attention over packed variable-length segments, with
    an optional local window (left, right) and softcap (see attn_fwd)."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    return _Attention.apply(q, k, v, cu_seqlens_q, cu_seqlens_k, int(max_seqlen_q),
                            int(max_seqlen_k), float(scale), bool(causal), window,
                            float(softcap or 0.0))
