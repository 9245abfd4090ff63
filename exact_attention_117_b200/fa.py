"""Python binding of the C ABI in include/fa.h (argument marshalling only).

Every step of the attention computation runs in the CUDA library
``libfa_b200.so``; this module only checks tensor properties, takes device
pointers and the current stream from torch, and turns status codes into
exceptions.  There is no fallback: if the library is missing or not built for
this GPU, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FA_LIBRARY selects another build of the same library (e.g. the bounds-checked
# libfa_b200_debug.so); by default the release build next to this file.
LIB_PATH = os.environ.get("FA_LIBRARY") or os.path.join(_HERE, "libfa_b200.so")

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK", 1: "FA_ERR_NULL", 2: "FA_ERR_SHAPE", 3: "FA_ERR_UNSUPPORTED_D",
    4: "FA_ERR_ALIGN", 5: "FA_ERR_SCALE", 6: "FA_ERR_WORKSPACE", 7: "FA_ERR_CUDA",
    8: "FA_ERR_DEVICE_TIMEOUT", 9: "FA_ERR_STATE",
}
KERNELS = ("fwd", "bwd_pre", "bwd_main", "bwd_dq", "fwd_combine", "fwd_kv_outer")

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.fa_status_string(status).decode() if _lib is not None else ""
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({msg})")


def load() -> ctypes.CDLL:
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run __graft_entry__.build())")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.restype = i
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    lib.fa_fwd_splitkv_workspace_size.restype = sz
    lib.fa_fwd_splitkv_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_fwd_splitkv.restype = i
    lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_fwd_kv_outer_workspace_size.restype = sz
    lib.fa_fwd_kv_outer_workspace_size.argtypes = [i, i, i, i]
    lib.fa_fwd_kv_outer.restype = i
    lib.fa_fwd_kv_outer.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd.restype = i
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, vp]
    lib.fa_bwd_deterministic.restype = i
    lib.fa_bwd_deterministic.argtypes = lib.fa_bwd.argtypes
    lib.fa_bwd_noalloc.restype = i
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    lib.fa_check_device_error.restype = i
    lib.fa_check_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
    lib.fa_selftest_watchdog.restype = i
    lib.fa_selftest_watchdog.argtypes = [ctypes.c_uint, vp]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_status_string.argtypes = [i]
    lib.fa_timing_begin.restype = i
    lib.fa_timing_begin.argtypes = []
    lib.fa_timing_end.restype = i
    lib.fa_timing_end.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]
    lib.fa_version.restype = i
    lib.fa_version.argtypes = []
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != FA_OK:
        raise FaError(status, where)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_qkv(*ts: torch.Tensor):
    ref = ts[0]
    if ref.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    for t in ts:
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("tensors must be contiguous bf16 CUDA tensors")
        if t.shape != ref.shape:
            raise ValueError("all tensors must have the same [B, H, N, d] shape")


def fwd_raw(q: int, k: int, v: int, o: int, lse: int, B: int, H: int, N: int, d: int,
            causal: bool, scale: float, stream: int) -> int:
    """Direct call of ``fa_fwd`` with raw pointers; returns the status code."""
    return load().fa_fwd(q, k, v, o, lse, B, H, N, d, int(bool(causal)), float(scale), stream)


def bwd_raw(q, k, v, o, lse, do, dq, dk, dv, ws, ws_bytes, B, H, N, d, causal, scale,
            stream) -> int:
    """Direct call of ``fa_bwd`` with raw pointers; returns the status code."""
    return load().fa_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, ws_bytes, B, H, N, d,
                         int(bool(causal)), float(scale), stream)


def workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load().fa_bwd_workspace_size(B, H, N, d))


def forward(q, k, v, causal: bool = False, scale: Optional[float] = None, out=None,
            lse=None, stream=None):
    """O, LSE = attention(q, k, v); all [B, H, N, d] bf16 on the GPU."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check(fwd_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, causal, scale,
                   _stream_ptr(stream)), "fa_fwd")
    return out, lse


def splitkv_workspace_size(B: int, H: int, N: int, d: int, num_splits: int) -> int:
    return int(load().fa_fwd_splitkv_workspace_size(B, H, N, d, num_splits))


def forward_splitkv(q, k, v, causal: bool = False, scale: Optional[float] = None,
                    num_splits: int = 2, out=None, lse=None, workspace=None, stream=None):
    """O, LSE through the split-KV forward (key range cut into ``num_splits``)."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = splitkv_workspace_size(B, H, N, d, num_splits)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(load().fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d,
                                 int(bool(causal)), float(scale), int(num_splits),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream_ptr(stream)), "fa_fwd_splitkv")
    return out, lse


def bwd_deterministic_raw(q, k, v, o, lse, do, dq, dk, dv, ws, ws_bytes, B, H, N, d, causal,
                          scale, stream) -> int:
    """Direct call of ``fa_bwd_deterministic`` with raw pointers; returns the status code."""
    return load().fa_bwd_deterministic(q, k, v, o, lse, do, dq, dk, dv, ws, ws_bytes, B, H, N, d,
                                       int(bool(causal)), float(scale), stream)


def kv_outer_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load().fa_fwd_kv_outer_workspace_size(B, H, N, d))


def forward_kv_outer(q, k, v, causal: bool = False, scale: Optional[float] = None, out=None,
                     lse=None, workspace=None, stream=None):
    """O, LSE through the KV-outer (FlashAttention-1 order) forward kernel."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = kv_outer_workspace_size(B, H, N, d)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(load().fa_fwd_kv_outer(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d,
                                  int(bool(causal)), float(scale), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  _stream_ptr(stream)), "fa_fwd_kv_outer")
    return out, lse


def backward(q, k, v, o, lse, do, causal: bool = False, scale: Optional[float] = None,
             dq=None, dk=None, dv=None, workspace=None, stream=None,
             deterministic: bool = False):
    """dQ, dK, dV of sum(dO * O); the fp32 workspace is allocated here if not given.

    ``deterministic=True`` calls ``fa_bwd_deterministic`` (dQ summed in a fixed
    order, bitwise reproducible) instead of ``fa_bwd`` (dQ summed by atomics)."""
    _check_qkv(q, k, v, o, do)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be a contiguous fp32 [B, H, N] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    need = workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    raw, name = (bwd_deterministic_raw, "fa_bwd_deterministic") if deterministic else \
        (bwd_raw, "fa_bwd")
    _check(raw(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
               _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
               B, H, N, d, causal, scale, _stream_ptr(stream)), name)
    return dq, dk, dv


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa.h


def bwd_noalloc_raw(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, causal, scale,
                    stream) -> int:
    """Direct call of ``fa_bwd_noalloc`` with raw pointers; returns the status code."""
    return load().fa_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d,
                                 int(bool(causal)), float(scale), stream)


def backward_noalloc(q, k, v, o, lse, do, causal: bool = False, scale: Optional[float] = None,
                     dq=None, dk=None, dv=None, stream=None):
    """Like ``backward`` but through ``fa_bwd_noalloc``: the library's own fixed
    scratch array replaces the workspace, so the C call allocates nothing.
    Problems needing more than ``NOALLOC_SCRATCH_BYTES`` of scratch raise
    FaError(FA_ERR_WORKSPACE).  (The outputs are allocated here by torch only if
    the caller does not pass them.)"""
    _check_qkv(q, k, v, o, do)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be a contiguous fp32 [B, H, N] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    _check(bwd_noalloc_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                           _ptr(dk), _ptr(dv), B, H, N, d, causal, scale, _stream_ptr(stream)),
           "fa_bwd_noalloc")
    return dq, dk, dv


def check_device_error(stream=None):
    """Synchronise and raise FaError if a kernel gave up on a bounded wait."""
    detail = ctypes.c_uint(0)
    st = load().fa_check_device_error(_stream_ptr(stream), ctypes.byref(detail))
    if st != FA_OK:
        raise FaError(st, f"device error word 0x{detail.value:x}")


def selftest_watchdog(limit_ms: int = 200, stream=None):
    """Launch the bounded-wait self-test kernel (see fa_selftest_watchdog)."""
    _check(load().fa_selftest_watchdog(int(limit_ms), _stream_ptr(stream)), "fa_selftest_watchdog")


class KernelTimer:
    """Context manager: per-kernel CUDA-event time of every launch inside it."""

    def __enter__(self):
        _check(load().fa_timing_begin(), "fa_timing_begin")
        return self

    def __exit__(self, *exc):
        ms = (ctypes.c_float * len(KERNELS))()
        cnt = (ctypes.c_int * len(KERNELS))()
        _check(load().fa_timing_end(ms, cnt), "fa_timing_end")
        self.ms = {k: float(ms[i]) for i, k in enumerate(KERNELS)}
        self.launches = {k: int(cnt[i]) for i, k in enumerate(KERNELS)}
        return False
