"""Inference-shaped forward (Nq queries against Nk keys, key range split over CTAs and
merged with the (m, l) rule) against the fp64 oracle on the same seeded inputs.  The
queries are the last Nq positions of the key sequence (causal: j <= i + Nk - Nq).  Same
tolerances as the dense path: O max-abs <= 1e-2 beyond output rounding, LSE <= 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_60_b200 import fa
from parity import LSE_ATOL, O_ATOL, compare_forward, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def make(B, H, Nq, Nk, d, dtype, seed, kv_range=None):
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g).to(dtype)
    k = torch.randn((B, H, Nk, d), generator=g).to(dtype)
    v = torch.randn((B, H, Nk, d), generator=g).to(dtype)
    kv = None
    if kv_range is not None:
        kv = torch.randint(kv_range[0], kv_range[1] + 1, (B,), generator=g, dtype=torch.int32)
    return q, k, v, kv


def run(q, k, v, kv, *, causal, splits):
    d = q.shape[-1]
    o, lse = fa.forward_splitkv(q.to(DEV), k.to(DEV), v.to(DEV), scale=d ** -0.5, causal=causal,
                                kv_len=None if kv is None else kv.to(DEV), num_splits=splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    return {"o": o.cpu(), "lse": lse.cpu()}


def reference(q, k, v, kv, causal):
    return oracle.attention(to_f64(q), to_f64(k), to_f64(v), scale=q.shape[-1] ** -0.5,
                            causal=causal, kv_len=None if kv is None else kv.numpy())


CASES = [
    # (B, H, Nq, Nk, d, dtype, causal, kv_range, splits, seed)
    (4, 4, 1, 4096, 128, torch.bfloat16, False, None, 0, 1),
    (2, 3, 1, 4096, 64, torch.bfloat16, True, (1, 4096), 7, 2),
    (2, 2, 16, 2000, 64, torch.float16, True, (1000, 2000), 0, 3),
    (1, 4, 130, 1024, 64, torch.bfloat16, True, None, 3, 4),
    (1, 2, 5, 129, 64, torch.bfloat16, False, None, 8, 5),
    (2, 2, 64, 3000, 128, torch.float16, False, (1, 3000), 0, 6),
    (1, 2, 200, 100, 64, torch.bfloat16, True, None, 0, 7),
    (1, 1, 333, 777, 128, torch.bfloat16, True, None, 2, 8),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype,causal,kvr,splits,seed", CASES)
def test_splitkv_matches_oracle(B, H, Nq, Nk, d, dtype, causal, kvr, splits, seed):
    q, k, v, kv = make(B, H, Nq, Nk, d, dtype, seed, kvr)
    gpu = run(q, k, v, kv, causal=causal, splits=splits)
    ref = reference(q, k, v, kv, causal)
    f = compare_forward(gpu, ref)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f


def test_split_count_does_not_change_the_result():
    q, k, v, kv = make(2, 2, 8, 5000, 64, torch.bfloat16, 11, (2500, 5000))
    outs = [run(q, k, v, kv, causal=True, splits=s) for s in (1, 2, 5, 16, 0)]
    for other in outs[1:]:
        assert torch.allclose(other["o"].float(), outs[0]["o"].float(), atol=4e-3, rtol=0)
        assert torch.allclose(other["lse"], outs[0]["lse"], atol=1e-4, rtol=0)


def test_square_single_split_is_the_dense_forward():
    q, k, v, kv = make(2, 3, 300, 300, 128, torch.bfloat16, 12, (100, 300))
    a = run(q, k, v, kv, causal=True, splits=1)
    o, lse = fa.forward(q.to(DEV), k.to(DEV), v.to(DEV), scale=128 ** -0.5, causal=True,
                        kv_len=kv.to(DEV))
    assert torch.equal(a["o"], o.cpu()) and torch.equal(a["lse"], lse.cpu())


def test_empty_key_set_gives_zero_output():
    q, k, v, _ = make(2, 2, 3, 500, 64, torch.bfloat16, 13)
    kv = torch.tensor([0, 400], dtype=torch.int32)
    gpu = run(q, k, v, kv, causal=False, splits=4)
    assert torch.all(gpu["o"][0] == 0) and torch.all(torch.isneginf(gpu["lse"][0]))
    ref = reference(q, k, v, kv, False)
    f = compare_forward(gpu, ref)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f


def test_long_context_decode_sampled_heads():
    """B8 H16, one query against 32K keys, d = 128 (decode against a long cache), auto
    splits: two heads against the oracle in full, the rest checked for finiteness."""
    q, k, v, _ = make(8, 16, 1, 32768, 128, torch.bfloat16, 14)
    gpu = run(q, k, v, None, causal=True, splits=0)
    heads = [(0, 0), (5, 11)]
    ref = oracle.attention(to_f64(q), to_f64(k), to_f64(v), scale=128 ** -0.5, causal=True,
                           heads=heads)
    mask = np.zeros((8, 16), bool)
    for b, h in heads:
        mask[b, h] = True
    f = compare_forward(gpu, ref, mask)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert torch.isfinite(gpu["o"].float()).all() and torch.isfinite(gpu["lse"]).all()
