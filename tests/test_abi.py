"""The C-ABI library loads, exports every entry point include/fa.h declares, and its
host-side argument checks reject bad calls before touching CUDA (no GPU needed)."""
import ctypes
import os
import re

import pytest

from exact_io_aware_60_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    with open(os.path.join(ROOT, "include", "fa.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"^FA_API\s+[\w\s\*]*?\b(fa_\w+)\s*\(", src, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_strerror",
              "fa_get_device_status", "fa_last_cuda_error", "fa_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fa.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_version_and_strerror():
    assert fa.fa_version() >= 100
    L = fa.lib()
    for code in range(5):
        assert L.fa_strerror(code).decode() == fa.fa_strerror(code)
    assert L.fa_strerror(99).decode() == "unknown status"


def test_workspace_bytes():
    L = fa.lib()
    n = L.fa_bwd_workspace_bytes(2, 3, 100, 64)
    r256 = lambda x: ((x + 255) // 256) * 256
    # fp32 dQ accumulator [B,H,N,d] + two fp32 [B,H,Npad] vectors (Npad = 128)
    assert n == r256(2 * 3 * 100 * 64 * 4) + 2 * r256(2 * 3 * 128 * 4)
    assert L.fa_bwd_workspace_bytes(0, 3, 100, 64) == 0


GOOD = dict(B=1, H=1, N=16, d=64, scale=0.125, causal=0, dtype=0)
P = 4096  # fake, 16-byte aligned non-null "device" address: never dereferenced


def call_fwd(**over):
    a = dict(GOOD, q=P, k=P, v=P, o=P, lse=P, kv=None)
    a.update(over)
    return fa.lib().fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"],
                           a["d"], a["scale"], a["causal"], a["kv"], a["dtype"], None)


@pytest.mark.parametrize("over,code", [
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(lse=None), fa.FA_ERR_INVALID_ARG),
    (dict(k=P + 8), fa.FA_ERR_INVALID_ARG),
    (dict(kv=P + 2), fa.FA_ERR_INVALID_ARG),
    (dict(B=0), fa.FA_ERR_INVALID_ARG),
    (dict(N=-1), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), fa.FA_ERR_INVALID_ARG),
    (dict(dtype=7), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
    (dict(B=1 << 16, H=1 << 15), fa.FA_ERR_UNSUPPORTED),
])
def test_fwd_rejects_bad_arguments_on_host(over, code):
    assert call_fwd(**over) == code


def call_bwd(**over):
    a = dict(GOOD, ptr=P, ws=P * 16, wsb=1 << 30, kv=None)
    a.update(over)
    p = a["ptr"]
    return fa.lib().fa_bwd(p, p, p, p, p, p, p, p, p, a["B"], a["H"], a["N"], a["d"],
                           a["scale"], a["causal"], a["kv"], a["dtype"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("over,code", [
    (dict(ptr=None), fa.FA_ERR_INVALID_ARG),
    (dict(ptr=P + 4), fa.FA_ERR_INVALID_ARG),
    (dict(ws=None), fa.FA_ERR_INVALID_ARG),
    (dict(ws=P * 16 + 16), fa.FA_ERR_INVALID_ARG),
    (dict(wsb=16), fa.FA_ERR_INVALID_ARG),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
])
def test_bwd_rejects_bad_arguments_on_host(over, code):
    assert call_bwd(**over) == code


def test_timing_hook_arguments():
    L = fa.lib()
    assert L.fa_set_timing_events(2, None, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_set_timing_events(0, P, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_set_timing_events(1, None, None) == fa.FA_OK


def test_binding_raises_without_cuda_tensors():
    import torch
    x = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(fa.FAError):
        fa.fa_fwd(x, x, x, x, torch.zeros(1, 1, 4), scale=0.1)


def test_blocksparse_rejects_missing_or_bad_mask():
    L = fa.lib()
    a = dict(GOOD)
    rc = L.fa_fwd_blocksparse(P, P, P, P, P, a["B"], a["H"], a["N"], a["d"], a["scale"], 0,
                              None, None, 0, 0, None)
    assert rc == fa.FA_ERR_INVALID_ARG
    rc = L.fa_fwd_blocksparse(P, P, P, P, P, a["B"], a["H"], a["N"], a["d"], a["scale"], 0,
                              None, P, 2, 0, None)
    assert rc == fa.FA_ERR_INVALID_ARG
    rc = L.fa_bwd_blocksparse(P, P, P, P, P, P, P, P, P, a["B"], a["H"], a["N"], a["d"],
                              a["scale"], 0, None, None, 0, 0, P * 16, 1 << 30, None)
    assert rc == fa.FA_ERR_INVALID_ARG


def call_fwd_dropout(p_drop, **over):
    a = dict(GOOD, q=P, k=P, v=P, o=P, lse=P, kv=None)
    a.update(over)
    return fa.lib().fa_fwd_dropout(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"],
                                   a["N"], a["d"], a["scale"], a["causal"], a["kv"], p_drop,
                                   1234, 0, a["dtype"], None)


def call_bwd_dropout(p_drop, **over):
    a = dict(GOOD, ws=P, ws_bytes=1 << 30, kv=None)
    a.update(over)
    return fa.lib().fa_bwd_dropout(P, P, P, P, P, P, P, P, P, a["B"], a["H"], a["N"], a["d"],
                                   a["scale"], a["causal"], a["kv"], p_drop, 1234, 0, a["dtype"],
                                   a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("p_drop", [float("nan"), float("inf"), -0.01, 255.6 / 256, 1.0, 3.0])
def test_dropout_rejects_bad_probability_on_host(p_drop):
    assert call_fwd_dropout(p_drop) == fa.FA_ERR_INVALID_ARG
    assert call_bwd_dropout(p_drop) == fa.FA_ERR_INVALID_ARG
    assert fa.lib().fa_dropout_mask(1, 1, 16, p_drop, 1, 0, P, None) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("over", [dict(q=None), dict(B=0), dict(scale=-1.0), dict(dtype=5)])
def test_dropout_forward_keeps_the_common_checks(over):
    assert call_fwd_dropout(0.1, **over) == fa.FA_ERR_INVALID_ARG


def test_dropout_backward_keeps_the_common_checks():
    assert call_bwd_dropout(0.1, ws_bytes=16) == fa.FA_ERR_INVALID_ARG
    assert call_bwd_dropout(0.1, ws=P + 16) == fa.FA_ERR_INVALID_ARG
    assert call_bwd_dropout(0.1, d=96) == fa.FA_ERR_UNSUPPORTED


def test_dropout_mask_rejects_bad_arguments_on_host():
    L = fa.lib()
    assert L.fa_dropout_mask(1, 1, 16, 0.1, 1, 0, None, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_dropout_mask(0, 1, 16, 0.1, 1, 0, P, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_dropout_mask(1, 1, 0, 0.1, 1, 0, P, None) == fa.FA_ERR_INVALID_ARG
    # more than FA_MAX_ELEMENTS (2^40) mask bytes
    assert L.fa_dropout_mask(1 << 10, 1, 1 << 16, 0.1, 1, 0, P, None) == fa.FA_ERR_INVALID_ARG


def test_splitkv_workspace_bytes():
    L = fa.lib()
    r256 = lambda x: ((x + 255) // 256) * 256
    # explicit splits: fp32 partial O [splits, B*H, Nq, d] + partial LSE [splits, B*H, Nq]
    assert L.fa_fwd_splitkv_workspace_bytes(2, 3, 5, 4096, 64, 4) == \
        r256(4 * 6 * 5 * 64 * 4) + r256(4 * 6 * 5 * 4)
    # one split needs no workspace; splits are capped by the key blocks (64 keys at d=64)
    assert L.fa_fwd_splitkv_workspace_bytes(2, 3, 5, 4096, 64, 1) == 0
    assert L.fa_fwd_splitkv_workspace_bytes(1, 1, 1, 100, 64, 8) == \
        r256(2 * 1 * 1 * 64 * 4) + r256(2 * 1 * 1 * 4)
    assert L.fa_fwd_splitkv_workspace_bytes(1, 1, 1, 100, 96, 8) == 0
    assert L.fa_fwd_splitkv_workspace_bytes(1, 1, 1, 100, 64, 10000) == 0


def _auto_splits(B, H, Nq, Nk, d):
    """Split count behind the automatic workspace size (1 when none is needed)."""
    r256 = lambda x: ((x + 255) // 256) * 256
    n = fa.lib().fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, 0)
    if n == 0:
        return 1
    found = [sp for sp in range(2, 129) if r256(sp * B * H * Nq * d * 4) + r256(sp * B * H * Nq * 4) == n]
    assert len(found) == 1, (n, found)
    return found[0]


def test_splitkv_automatic_split_count():
    # decode (one query tile per head, fewer tiles than SMs): the keys are split, into
    # pieces of at least two key blocks, and never more than 128 of them
    for B, H, Nk, d in ((8, 16, 32768, 128), (1, 8, 131072, 64), (2, 2, 5000, 64)):
        sp = _auto_splits(B, H, 1, Nk, d)
        bn = 64 if d == 64 else 128
        kblocks = -(-Nk // bn)
        assert 1 < sp <= 128 and -(-kblocks // sp) >= 2, (B, H, Nk, d, sp)
    # many query tiles per SM already: no split
    assert _auto_splits(64, 32, 512, 4096, 64) == 1
    # too few key blocks to split
    assert _auto_splits(1, 1, 1, 200, 128) == 1


def call_splitkv(**over):
    a = dict(GOOD, Nq=4, Nk=64, q=P, k=P, v=P, o=P, lse=P, kv=None, splits=0, ws=P,
             ws_bytes=1 << 30)
    a.update(over)
    return fa.lib().fa_fwd_splitkv(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"],
                                   a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"], a["kv"],
                                   a["splits"], a["dtype"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("over,code", [
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(k=P + 4), fa.FA_ERR_INVALID_ARG),
    (dict(Nk=0), fa.FA_ERR_INVALID_ARG),
    (dict(Nq=0), fa.FA_ERR_INVALID_ARG),
    (dict(splits=-1), fa.FA_ERR_INVALID_ARG),
    (dict(splits=257), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(d=80), fa.FA_ERR_UNSUPPORTED),
])
def test_splitkv_rejects_bad_arguments_on_host(over, code):
    assert call_splitkv(**over) == code


def call_fp8(**over):
    a = dict(GOOD, d=128, q=P, k=P, v=P, o=P, lse=P, kv=None, qs=0.5, ks=0.5, vs=0.5)
    a.update(over)
    return fa.lib().fa_fwd_fp8(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"],
                               a["d"], a["scale"], a["causal"], a["kv"], a["qs"], a["ks"],
                               a["vs"], None)


@pytest.mark.parametrize("over,code", [
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(v=P + 8), fa.FA_ERR_INVALID_ARG),
    (dict(qs=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(ks=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(vs=-1.0), fa.FA_ERR_INVALID_ARG),
    (dict(N=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=64), fa.FA_ERR_UNSUPPORTED),
])
def test_fp8_rejects_bad_arguments_on_host(over, code):
    assert call_fp8(**over) == code
