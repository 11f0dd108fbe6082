"""ctypes binding of libfa.so (declared in include/fa.h).

The functions named like the C entry points (``fa_fwd``, ``fa_bwd``, ...) only marshal
arguments: they check shapes and dtypes, take raw device pointers from torch tensors
and pass the current CUDA stream.  Every step of the computation runs in the library's
CUDA kernels.  ``forward`` / ``backward`` additionally allocate the outputs with torch.

The library is loaded on first use.  If ``libfa.so`` is missing, or a call returns an
error, a :class:`FAError` is raised: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)
FA_ERR_SCRATCH_LIMIT = 5
FA_NOALLOC_SCRATCH_BYTES = 64 << 20
FA_BF16, FA_FP16 = 0, 1

_lock = threading.Lock()
_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if _lib is not None:
            detail = _lib.fa_last_cuda_error().decode()
        msg = f"{where}: {fa_strerror(status)} (status {status})"
        if status == FA_ERR_CUDA and detail:
            msg += f": {detail}"
        super().__init__(msg)


def lib():
    """The loaded ctypes library (raises if libfa.so has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise FAError(FA_ERR_UNSUPPORTED,
                              f"libfa.so not found at {LIB_PATH} (build it with "
                              "`python -m exact_io_aware_60_b200.build`)")
            L = ctypes.CDLL(LIB_PATH)
            vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            L.fa_fwd.restype = i
            L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, i, vp]
            L.fa_bwd.restype = i
            L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, i,
                                 vp, sz, vp]
            L.fa_bwd_workspace_bytes.restype = sz
            L.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
            L.fa_strerror.restype = ctypes.c_char_p
            L.fa_strerror.argtypes = [i]
            L.fa_last_cuda_error.restype = ctypes.c_char_p
            L.fa_last_cuda_error.argtypes = []
            L.fa_get_device_status.restype = i
            L.fa_get_device_status.argtypes = [vp]
            L.fa_version.restype = i
            L.fa_version.argtypes = []
            L.fa_set_timing_events.restype = i
            L.fa_set_timing_events.argtypes = [i, vp, vp]
            L.fa_selftest_wait_timeout.restype = i
            L.fa_selftest_wait_timeout.argtypes = [i, vp]
            L.fa_fwd_blocksparse.restype = i
            L.fa_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp, i, i,
                                             vp]
            L.fa_bwd_blocksparse.restype = i
            L.fa_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f,
                                             i, vp, vp, i, i, vp, sz, vp]
            u64, u32 = ctypes.c_ulonglong, ctypes.c_uint
            L.fa_fwd_dropout.restype = i
            L.fa_fwd_dropout.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, f, u64, u32, i,
                                         vp]
            L.fa_bwd_dropout.restype = i
            L.fa_bwd_dropout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp,
                                         f, u64, u32, i, vp, sz, vp]
            L.fa_dropout_mask.restype = i
            L.fa_dropout_mask.argtypes = [i, i, i, f, u64, u32, vp, vp]
            L.fa_fwd_splitkv_workspace_bytes.restype = sz
            L.fa_fwd_splitkv_workspace_bytes.argtypes = [i, i, i, i, i, i]
            L.fa_fwd_splitkv.restype = i
            L.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, i, i, vp, sz,
                                         vp]
            L.fa_fwd_fp8.restype = i
            L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, f, f, f, vp]
            L.fa_bwd_noalloc.restype = i
            L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i,
                                         vp, i, vp]
            L.fa_schedule_items.restype = i
            L.fa_schedule_items.argtypes = [vp, i, i, vp, vp]
            _lib = L
    return _lib


def fa_strerror(status: int) -> str:
    if _lib is None:
        return {0: "ok", 1: "invalid argument", 2: "unsupported configuration or device",
                3: "CUDA error", 4: "device-side wait timed out",
                5: "problem needs more scratch than fa_bwd_noalloc's static buffer"}.get(
                    status, "unknown status")
    return _lib.fa_strerror(int(status)).decode()


def fa_version() -> int:
    return int(lib().fa_version())


def fa_schedule_items(cost, lists: int):
    """The launchers' static schedule of items with host costs ``cost`` over ``lists``
    lists: (off, ids) as numpy arrays, list c = ids[off[c]:off[c + 1]] (host only)."""
    import numpy as np
    c = np.ascontiguousarray(np.asarray(cost, dtype=np.float32))
    off = np.zeros(int(lists) + 1, dtype=np.uint16)
    ids = np.zeros(max(len(c), 1), dtype=np.uint16)
    rc = lib().fa_schedule_items(c.ctypes.data, len(c), int(lists), off.ctypes.data,
                                 ids.ctypes.data)
    if rc != FA_OK:
        raise FAError(rc, "fa_schedule_items")
    return off, ids[:len(c)]


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise FAError(FA_ERR_INVALID_ARG, f"unsupported dtype {t.dtype}")


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check(t: torch.Tensor, name: str, shape, dtype):
    if not isinstance(t, torch.Tensor):
        raise FAError(FA_ERR_INVALID_ARG, f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise FAError(FA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise FAError(FA_ERR_INVALID_ARG,
                      f"{name}: expected contiguous {dtype} {tuple(shape)}, got "
                      f"{t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()}")


def _kv_ptr(kv_len, B):
    if kv_len is None:
        return None
    _check(kv_len, "kv_len", (B,), torch.int32)
    return kv_len.data_ptr()


def fa_fwd(q, k, v, o, lse, *, scale: float, causal: bool = False, kv_len=None,
           stream=None) -> None:
    """Enqueues the forward pass: writes ``o`` ([B,H,N,d]) and ``lse`` ([B,H,N] fp32)."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check(t, name, (B, H, N, d), q.dtype)
    _check(lse, "lse", (B, H, N), torch.float32)
    rc = lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      B, H, N, d, float(scale), int(bool(causal)), _kv_ptr(kv_len, B),
                      _dtype_code(q), _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd")


def fa_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_bytes(B, H, N, d))


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, *, scale: float, causal: bool = False,
           kv_len=None, workspace: torch.Tensor, stream=None) -> None:
    """Enqueues the backward pass: writes ``dq``, ``dk``, ``dv``.  ``workspace`` is a
    uint8 CUDA tensor of at least ``fa_bwd_workspace_bytes`` bytes."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq),
                    ("dk", dk), ("dv", dv)):
        _check(t, name, (B, H, N, d), q.dtype)
    _check(lse, "lse", (B, H, N), torch.float32)
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise FAError(FA_ERR_INVALID_ARG, "workspace must be a contiguous uint8 CUDA tensor")
    rc = lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                      lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                      float(scale), int(bool(causal)), _kv_ptr(kv_len, B), _dtype_code(q),
                      workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd")


def _mask_args(block_mask, B, H, N):
    T = (N + 127) // 128
    if not isinstance(block_mask, torch.Tensor) or not block_mask.is_cuda:
        raise FAError(FA_ERR_INVALID_ARG, "block_mask must be a CUDA tensor")
    if block_mask.dtype != torch.uint8 or not block_mask.is_contiguous():
        raise FAError(FA_ERR_INVALID_ARG, "block_mask must be a contiguous uint8 tensor")
    if tuple(block_mask.shape) == (T, T):
        return block_mask.data_ptr(), 0
    if tuple(block_mask.shape) == (B, H, T, T):
        return block_mask.data_ptr(), 1
    raise FAError(FA_ERR_INVALID_ARG,
                  f"block_mask shape must be ({T}, {T}) or ({B}, {H}, {T}, {T})")


def fa_fwd_blocksparse(q, k, v, o, lse, block_mask, *, scale: float, causal: bool = False,
                       kv_len=None, stream=None) -> None:
    """Block-sparse forward: ``block_mask`` is a uint8 CUDA tensor [T, T] or [B, H, T, T]
    (T = ceil(N/128)); key tile kt is visible to query tile qt only where it is nonzero."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check(t, name, (B, H, N, d), q.dtype)
    _check(lse, "lse", (B, H, N), torch.float32)
    mp, per_head = _mask_args(block_mask, B, H, N)
    rc = lib().fa_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), B, H, N, d, float(scale), int(bool(causal)),
                                  _kv_ptr(kv_len, B), mp, per_head, _dtype_code(q),
                                  _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_blocksparse")


def fa_bwd_blocksparse(q, k, v, o, dout, lse, dq, dk, dv, block_mask, *, scale: float,
                       causal: bool = False, kv_len=None, workspace: torch.Tensor,
                       stream=None) -> None:
    """Block-sparse backward with the same ``block_mask`` as the forward call."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq),
                    ("dk", dk), ("dv", dv)):
        _check(t, name, (B, H, N, d), q.dtype)
    _check(lse, "lse", (B, H, N), torch.float32)
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise FAError(FA_ERR_INVALID_ARG, "workspace must be a contiguous uint8 CUDA tensor")
    mp, per_head = _mask_args(block_mask, B, H, N)
    rc = lib().fa_bwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                  dv.data_ptr(), B, H, N, d, float(scale), int(bool(causal)),
                                  _kv_ptr(kv_len, B), mp, per_head, _dtype_code(q),
                                  workspace.data_ptr(), workspace.numel(),
                                  _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_blocksparse")


def fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, *, scale: float, causal: bool = False,
                   kv_len=None, stream=None) -> None:
    """Enqueues the backward pass using the library's static scratch instead of a
    caller workspace, for callers that cannot allocate device memory (see include/fa.h:
    problems needing more than FA_NOALLOC_SCRATCH_BYTES of scratch are refused, and
    calls that may overlap on the GPU race on the shared scratch)."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq),
                    ("dk", dk), ("dv", dv)):
        _check(t, name, (B, H, N, d), q.dtype)
    _check(lse, "lse", (B, H, N), torch.float32)
    rc = lib().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), B, H, N, d, float(scale), int(bool(causal)),
                              _kv_ptr(kv_len, B), _dtype_code(q), _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_noalloc")


def fa_fwd_dropout(q, k, v, o, lse, *, scale: float, p_drop: float, seed: int, offset: int = 0,
                   causal: bool = False, kv_len=None, stream=None) -> None:
    """Forward pass with dropout of probability ``p_drop`` on the attention weights; the
    keep mask is drawn from (``seed``, ``offset``) and never stored (see include/fa.h)."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check(t, name, (B, H, N, d), q.dtype)
    _check(lse, "lse", (B, H, N), torch.float32)
    rc = lib().fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), B, H, N, d, float(scale), int(bool(causal)),
                              _kv_ptr(kv_len, B), float(p_drop), int(seed), int(offset),
                              _dtype_code(q), _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_dropout")


def fa_bwd_dropout(q, k, v, o, dout, lse, dq, dk, dv, *, scale: float, p_drop: float, seed: int,
                   offset: int = 0, causal: bool = False, kv_len=None, workspace: torch.Tensor,
                   stream=None) -> None:
    """Backward pass of :func:`fa_fwd_dropout`; give it the same p_drop, seed, offset."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq),
                    ("dk", dk), ("dv", dv)):
        _check(t, name, (B, H, N, d), q.dtype)
    _check(lse, "lse", (B, H, N), torch.float32)
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise FAError(FA_ERR_INVALID_ARG, "workspace must be a contiguous uint8 CUDA tensor")
    rc = lib().fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), B, H, N, d, float(scale), int(bool(causal)),
                              _kv_ptr(kv_len, B), float(p_drop), int(seed), int(offset),
                              _dtype_code(q), workspace.data_ptr(), workspace.numel(),
                              _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_dropout")


def fa_dropout_mask(keep, *, p_drop: float, seed: int, offset: int = 0, stream=None) -> None:
    """Writes the keep mask of the dropout calls into ``keep``, a uint8 CUDA tensor
    [B, H, N, N] (1 = kept)."""
    if not isinstance(keep, torch.Tensor) or not keep.is_cuda or keep.dtype != torch.uint8 \
            or not keep.is_contiguous() or keep.dim() != 4 or keep.shape[2] != keep.shape[3]:
        raise FAError(FA_ERR_INVALID_ARG, "keep must be a contiguous uint8 CUDA tensor [B,H,N,N]")
    B, H, N, _ = keep.shape
    rc = lib().fa_dropout_mask(B, H, N, float(p_drop), int(seed), int(offset), keep.data_ptr(),
                               _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_dropout_mask")


def fa_fwd_splitkv_workspace_bytes(B: int, H: int, Nq: int, Nk: int, d: int,
                                   num_splits: int = 0) -> int:
    return int(lib().fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, num_splits))


def fa_fwd_splitkv(q, k, v, o, lse, *, scale: float, causal: bool = False, kv_len=None,
                   num_splits: int = 0, workspace=None, stream=None) -> None:
    """Inference-shaped forward: q, o [B,H,Nq,d] against k, v [B,H,Nk,d], the key range
    split over CTAs and merged (see include/fa.h).  ``workspace``: uint8 CUDA tensor of
    ``fa_fwd_splitkv_workspace_bytes`` bytes (None allowed when that is 0)."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    for name, t, n in (("q", q, Nq), ("k", k, Nk), ("v", v, Nk), ("o", o, Nq)):
        _check(t, name, (B, H, n, d), q.dtype)
    _check(lse, "lse", (B, H, Nq), torch.float32)
    if workspace is not None and (not workspace.is_cuda or workspace.dtype != torch.uint8
                                  or not workspace.is_contiguous()):
        raise FAError(FA_ERR_INVALID_ARG, "workspace must be a contiguous uint8 CUDA tensor")
    rc = lib().fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), B, H, Nq, Nk, d, float(scale), int(bool(causal)),
                              _kv_ptr(kv_len, B), int(num_splits), _dtype_code(q),
                              None if workspace is None else workspace.data_ptr(),
                              0 if workspace is None else workspace.numel(),
                              _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_splitkv")


def forward_splitkv(q, k, v, *, scale: Optional[float] = None, causal: bool = False,
                    kv_len=None, num_splits: int = 0, stream=None):
    """Allocates ``o``, ``lse`` and the workspace with torch and runs :func:`fa_fwd_splitkv`."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    B, H, Nq, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    n = fa_fwd_splitkv_workspace_bytes(B, H, Nq, k.shape[2], d, num_splits)
    ws = torch.empty(n, dtype=torch.uint8, device=q.device) if n > 0 else None
    fa_fwd_splitkv(q, k, v, o, lse, scale=scale, causal=causal, kv_len=kv_len,
                   num_splits=num_splits, workspace=ws, stream=stream)
    return o, lse


def fa_fwd_fp8(q8, k8, v8, o, lse, *, scale: float, q_scale: float, k_scale: float,
               v_scale: float, causal: bool = False, kv_len=None, stream=None) -> None:
    """FP8 forward: q8, k8, v8 are E4M3 tensors (torch.float8_e4m3fn, or their uint8 bytes)
    [B,H,N,128] with per-tensor scale factors; writes bf16 ``o`` and fp32 ``lse``."""
    B, H, N, d = q8.shape
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        if not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, H, N, d) \
                or t.element_size() != 1:
            raise FAError(FA_ERR_INVALID_ARG, f"{name} must be a contiguous 1-byte CUDA tensor "
                                              f"of shape {(B, H, N, d)}")
    _check(o, "o", (B, H, N, d), torch.bfloat16)
    _check(lse, "lse", (B, H, N), torch.float32)
    rc = lib().fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), o.data_ptr(),
                          lse.data_ptr(), B, H, N, d, float(scale), int(bool(causal)),
                          _kv_ptr(kv_len, B), float(q_scale), float(k_scale), float(v_scale),
                          _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_fp8")


def fa_set_timing_events(which: int, start=None, stop=None) -> None:
    """Profiling hook: record torch.cuda.Event ``start``/``stop`` around every launch of
    the forward kernel (which=0) or the backward main kernel (which=1); None switches it
    off.  The events must have been recorded once (so that they exist)."""
    h0 = None if start is None else start.cuda_event
    h1 = None if stop is None else stop.cuda_event
    rc = lib().fa_set_timing_events(int(which), h0, h1)
    if rc != FA_OK:
        raise FAError(rc, "fa_set_timing_events")


def fa_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Enqueues the bounded-wait self-test kernel (see include/fa.h)."""
    rc = lib().fa_selftest_wait_timeout(int(limit_us), _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, "fa_selftest_wait_timeout")


def fa_get_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status word."""
    return int(lib().fa_get_device_status(_stream_handle(stream)))


# ------------------------------------------------------------------ conveniences

def forward(q, k, v, *, scale: Optional[float] = None, causal: bool = False, kv_len=None,
            stream=None):
    """Allocates ``o`` and ``lse`` with torch and runs :func:`fa_fwd`."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    fa_fwd(q, k, v, o, lse, scale=scale, causal=causal, kv_len=kv_len, stream=stream)
    return o, lse


def workspace_for(q) -> torch.Tensor:
    B, H, N, d = q.shape
    return torch.empty(fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)


def backward(q, k, v, o, dout, lse, *, scale: Optional[float] = None, causal: bool = False,
             kv_len=None, workspace=None, stream=None):
    """Allocates ``dq``, ``dk``, ``dv`` (and the workspace if not given) and runs
    :func:`fa_bwd`."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        workspace = workspace_for(q)
    fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, scale=scale, causal=causal, kv_len=kv_len,
           workspace=workspace, stream=stream)
    return dq, dk, dv
