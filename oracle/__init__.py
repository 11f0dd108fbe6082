"""fp64 CPU oracle for exact attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code with the
CUDA library under ``exact_io_aware_60_b200/`` and imports nothing from it.

The arithmetic lives in ``attn_oracle.c``: the plain definition of standard attention
(score matrix materialised, textbook softmax, textbook chain rule), which FlashAttention
reproduces exactly up to floating-point ordering (anthology note "NOTE-005:
FlashAttention", Theorem 1; promptingindex page "FlashAttention: The IO-Aware Algorithm
That Rewrote GPU Training Speed Records", section "Tiling").  This module only marshals
numpy arrays into it.

Pins: every function here is pinned by ``tests/test_oracle_pins.py`` (brute-force
softmax without max shift, closed forms, invariants, central finite differences) and,
for dropout and its random numbers, by ``tests/test_oracle_dropout_pins.py`` (published
Philox4x32-10 known-answer vectors, cuRAND's host Philox generator, statistics of the
mask, finite differences through a fixed mask).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` into ``liboracle.so`` (gcc, OpenMP, portable -O3)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-fPIC", "-shared", "-fopenmp", "-std=c11", "-Wall",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Dropout(ctypes.Structure):
    _fields_ = [("threshold", ctypes.c_uint), ("seed", ctypes.c_ulonglong),
                ("offset", ctypes.c_uint), ("bh", ctypes.c_uint)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            lp = ctypes.POINTER(ctypes.c_long)
            lib.oracle_attention_rows.restype = ctypes.c_int
            lib.oracle_attention_rows.argtypes = [
                dp, dp, dp, dp, ctypes.c_long, ctypes.c_long, ctypes.c_double, ctypes.c_int,
                ctypes.c_long, lp, ctypes.c_long, dp, dp, dp, dp, dp]
            lib.oracle_attention_rows_masked.restype = ctypes.c_int
            lib.oracle_attention_rows_masked.argtypes = [
                dp, dp, dp, dp, ctypes.c_long, ctypes.c_long, ctypes.c_double, ctypes.c_int,
                ctypes.c_long, ctypes.c_void_p, ctypes.c_long, lp, ctypes.c_long, dp, dp, dp,
                dp, dp]
            lib.oracle_attention_rows_ex.restype = ctypes.c_int
            lib.oracle_attention_rows_ex.argtypes = [
                dp, dp, dp, dp, ctypes.c_long, ctypes.c_long, ctypes.c_double, ctypes.c_int,
                ctypes.c_long, ctypes.c_void_p, ctypes.c_long, ctypes.POINTER(_Dropout), lp,
                ctypes.c_long, dp, dp, dp, dp, dp]
            lib.oracle_attention_rows_qk.restype = ctypes.c_int
            lib.oracle_attention_rows_qk.argtypes = [
                dp, dp, dp, dp, ctypes.c_long, ctypes.c_long, ctypes.c_long, ctypes.c_double,
                ctypes.c_int, ctypes.c_long, ctypes.c_void_p, ctypes.c_long,
                ctypes.POINTER(_Dropout), lp, ctypes.c_long, dp, dp, dp, dp, dp]
            u32p = ctypes.POINTER(ctypes.c_uint)
            lib.oracle_philox4x32_10.restype = None
            lib.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
            lib.oracle_dropout_byte.restype = ctypes.c_uint
            lib.oracle_dropout_byte.argtypes = [ctypes.c_ulonglong, ctypes.c_uint, ctypes.c_uint,
                                                ctypes.c_long, ctypes.c_long]
            lib.oracle_dropout_keep.restype = ctypes.c_int
            lib.oracle_dropout_keep.argtypes = [ctypes.c_uint, ctypes.c_ulonglong, ctypes.c_uint,
                                                ctypes.c_uint, ctypes.c_long, ctypes.c_long,
                                                ctypes.c_void_p]
            lib.oracle_threads.restype = ctypes.c_int
            lib.oracle_threads.argtypes = []
            lib.oracle_set_threads.restype = None
            lib.oracle_set_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_threads())


def set_threads(n: int) -> None:
    """OpenMP threads for later oracle calls (timing only; results do not depend on it
    beyond the order of the dK/dV sums)."""
    _load().oracle_set_threads(int(n))


def dropout_threshold(p) -> int:
    """Byte threshold t of drop probability ``p``: p is taken in single precision and
    rounded to the nearest multiple of 1/256 (ties to even); a random byte below t drops
    the element, so the drop probability used is exactly t / 256.  Valid for 0 <= t < 256.
    """
    t = int(np.rint(np.float32(p) * np.float32(256.0)))
    if not (0 <= t < 256):
        raise ValueError(f"dropout probability {p} is outside [0, 255.5/256)")
    return t


def philox4x32_10(ctr, key):
    """The four 32-bit output words of Philox4x32-10 for counter ``ctr`` (4 words) and
    key ``key`` (2 words)."""
    c = (ctypes.c_uint * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
    k = (ctypes.c_uint * 2)(*[int(x) & 0xFFFFFFFF for x in key])
    o = (ctypes.c_uint * 4)()
    _load().oracle_philox4x32_10(c, k, o)
    return [int(x) for x in o]


def dropout_byte(seed, offset, bh, i, j) -> int:
    """The random byte that decides element (i, j) of head ``bh``."""
    return int(_load().oracle_dropout_byte(int(seed), int(offset), int(bh), int(i), int(j)))


def dropout_keep(p, seed, offset, bh, n_q, n_k):
    """Keep mask ``[n_q, n_k]`` (uint8, 1 = kept) of head ``bh`` (= b * H + h)."""
    keep = np.zeros((n_q, n_k), dtype=np.uint8)
    rc = _load().oracle_dropout_keep(dropout_threshold(p), int(seed), int(offset), int(bh),
                                     n_q, n_k, keep.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise RuntimeError(f"oracle_dropout_keep failed with status {rc}")
    return keep


def _f64(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def attention_rows(q, k, v, dout=None, *, scale, causal=False, kv_len=None, rows=None,
                   want_dkdv=True, block_mask=None, block_size=128, dropout_p=0.0, seed=0,
                   offset=0, bh=0):
    """Exact attention of one (batch, head) for the query rows ``rows``.

    q, dout: ``[Nq, d]``; k, v: ``[Nk, d]`` (cast to fp64).  With Nq != Nk the queries are
    the last Nq positions of the key sequence (causal: key j visible to query i when
    j <= i + Nk - Nq).  ``kv_len``: valid keys (None = Nk).
    ``block_mask``: optional ``[nb, nb]`` array (nb = ceil(N / block_size)); key j is
    visible to query i only where ``block_mask[i // block_size, j // block_size]`` != 0.
    ``dropout_p``, ``seed``, ``offset``, ``bh``: dropout on the probabilities with the
    counter-based mask of head ``bh`` (see ``dropout_keep``); 0 = no dropout.
    Returns a dict with ``o [R,d]``, ``lse [R]`` and, when ``dout`` is given, ``dq [R,d]``
    and (if ``want_dkdv``) ``dk``, ``dv [N,d]`` summed over the given rows only.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    Nq, d = q.shape
    N = k.shape[0]
    assert k.shape == (N, d) and v.shape == (N, d)
    L = N if kv_len is None else int(kv_len)
    if rows is None:
        rows = np.arange(Nq, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    R = rows.shape[0]
    o = np.zeros((R, d))
    lse = np.zeros((R,))
    dq = dk = dv = None
    if dout is not None:
        dout = _f64(dout)
        assert dout.shape == (Nq, d)
        dq = np.zeros((R, d))
        if want_dkdv:
            dk = np.zeros((N, d))
            dv = np.zeros((N, d))
    mask_arr = None
    if block_mask is not None:
        nb = (N + block_size - 1) // block_size
        mask_arr = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
        assert mask_arr.shape == (nb, nb), (mask_arr.shape, nb)
    drop = _Dropout(dropout_threshold(dropout_p), int(seed), int(offset), int(bh))
    rc = _load().oracle_attention_rows_qk(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), Nq, N, d, float(scale), int(bool(causal)), L,
        None if mask_arr is None else mask_arr.ctypes.data_as(ctypes.c_void_p),
        int(block_size), ctypes.byref(drop), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
        R, _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_rows failed with status {rc}")
    out = {"o": o, "lse": lse}
    if dout is not None:
        out["dq"] = dq
        if want_dkdv:
            out["dk"] = dk
            out["dv"] = dv
    return out


def attention(q, k, v, dout=None, *, scale, causal=False, kv_len=None, heads=None,
              block_mask=None, block_size=128, dropout_p=0.0, seed=0, offset=0):
    """Exact attention over ``[B, H, N, d]`` arrays, one (b, h) at a time (k, v may be
    ``[B, H, Nk, d]`` with Nk != N: see ``attention_rows``).

    ``kv_len``: per-batch valid key counts (length B) or None.  ``heads``: optional list
    of (b, h) pairs to evaluate; the others are left as NaN in the outputs.
    ``block_mask``: optional ``[nb, nb]`` (shared by all heads) or ``[B, H, nb, nb]``.
    ``dropout_p``, ``seed``, ``offset``: dropout, head (b, h) drawing its mask as bh = b*H+h.
    Returns ``o``, ``lse`` and, with ``dout``, ``dq``, ``dk``, ``dv`` as fp64 arrays.
    """
    q = np.asarray(q)
    B, H, N, d = q.shape
    Nk = np.asarray(k).shape[2]
    o = np.full((B, H, N, d), np.nan)
    lse = np.full((B, H, N), np.nan)
    res = {"o": o, "lse": lse}
    if dout is not None:
        res["dq"] = np.full((B, H, N, d), np.nan)
        for name in ("dk", "dv"):
            res[name] = np.full((B, H, Nk, d), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        L = None if kv_len is None else int(kv_len[b])
        bm = None
        if block_mask is not None:
            bm = np.asarray(block_mask)
            bm = bm if bm.ndim == 2 else bm[b, h]
        r = attention_rows(q[b, h], k[b, h], v[b, h], None if dout is None else dout[b, h],
                           scale=scale, causal=causal, kv_len=L, block_mask=bm,
                           block_size=block_size, dropout_p=dropout_p, seed=seed, offset=offset,
                           bh=b * H + h)
        o[b, h] = r["o"]
        lse[b, h] = r["lse"]
        if dout is not None:
            res["dq"][b, h] = r["dq"]
            res["dk"][b, h] = r["dk"]
            res["dv"][b, h] = r["dv"]
    return res
