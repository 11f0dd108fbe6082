"""Dropout on the GPU: the keep mask bit for bit, and the fused forward / backward
against the fp64 oracle with the same (p, seed, offset).

The mask is integer work, so it is compared exactly: through fa_dropout_mask, and inside
the fused kernels by inputs that make every mask bit visible in the outputs (Q = 0 gives
uniform probabilities; one-hot rows of V, or of dO, then read the kept keys out of O, or
the kept queries out of dV).  The floating-point results use the dense tolerances, with O
graded as O / r (r = 1 / (1 - p), the factor that scales every kept weight, and with it
every rounding error of the weights), plus half an ulp of the output itself."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_60_b200 import fa
from exact_io_aware_60_b200 import workloads as W
from parity import GRAD_REL_L2, LSE_ATOL, O_ATOL, compare_backward, compare_forward, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def oracle_mask(B, H, N, p, seed, offset):
    return np.stack([oracle.dropout_keep(p, seed, offset, bh, N, N) for bh in range(B * H)]
                    ).reshape(B, H, N, N)


@pytest.mark.parametrize("B,H,N,p,seed,offset", [
    (1, 1, 16, 0.5, 0, 0),
    (2, 3, 200, 0.1, 1234, 0),
    (1, 2, 333, 0.9, (1 << 40) + 17, 5),
    (2, 1, 64, 255 / 256, 7, 1 << 31),
    (1, 1, 50, 0.0, 3, 0),
])
def test_mask_bit_exact(B, H, N, p, seed, offset):
    keep = torch.empty((B, H, N, N), dtype=torch.uint8, device=DEV)
    fa.fa_dropout_mask(keep, p_drop=p, seed=seed, offset=offset)
    torch.cuda.synchronize()
    ref = oracle_mask(B, H, N, p, seed, offset)
    assert np.array_equal(keep.cpu().numpy(), ref)


def keep_scale(p):
    """The library's r = 256 / (256 - t), t = rint(256 p): the multiplier of kept weights."""
    return 256.0 / (256 - int(np.rint(256 * p)))


def run_dropout(q, k, v, do, *, scale, causal, kv_len, p, seed, offset, backward=True):
    q, k, v = (t.to(DEV) for t in (q, k, v))
    kv = None if kv_len is None else kv_len.to(DEV)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=DEV)
    fa.fa_fwd_dropout(q, k, v, o, lse, scale=scale, causal=causal, kv_len=kv, p_drop=p,
                      seed=seed, offset=offset)
    out = {"o": o, "lse": lse}
    if backward:
        do = do.to(DEV)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        fa.fa_bwd_dropout(q, k, v, o, do, lse, dq, dk, dv, scale=scale, causal=causal,
                          kv_len=kv, p_drop=p, seed=seed, offset=offset,
                          workspace=fa.workspace_for(q))
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    return {n: t.cpu() for n, t in out.items()}


@pytest.mark.parametrize("d,N,causal,dtype", [(64, 64, False, torch.bfloat16),
                                              (64, 64, True, torch.float16),
                                              (128, 128, False, torch.float16),
                                              (128, 100, True, torch.bfloat16),
                                              (64, 300, False, torch.bfloat16),
                                              (128, 517, True, torch.bfloat16)])
def test_forward_mask_read_out_exactly(d, N, causal, dtype):
    """Q = 0 makes P_ij = 1 / L_i over the visible keys; with V_j = e_(j mod d),
    O_ic L_i / r counts the kept visible keys j = c (mod d) of row i."""
    B, H, p, seed, off = 2, 2, 0.3, 99, 3
    t = oracle.dropout_threshold(p)
    r = 256 / (256 - t)
    q = torch.zeros((B, H, N, d), dtype=dtype)
    k = torch.randn((B, H, N, d)).to(dtype)
    v = torch.zeros((B, H, N, d), dtype=dtype)
    v[:, :, torch.arange(N), torch.arange(N) % d] = 1
    gpu = run_dropout(q, k, v, None, scale=0.125, causal=causal, kv_len=None, p=p, seed=seed,
                      offset=off, backward=False)
    keep = oracle_mask(B, H, N, p, seed, off).astype(np.int64)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    vis = (j <= i) if causal else np.ones((N, N), bool)
    L = vis.sum(axis=1)
    counts = np.zeros((B, H, N, d), np.int64)
    for c in range(d):
        counts[..., c] = (keep * vis)[..., j[0] % d == c].sum(axis=-1)
    got = to_f64(gpu["o"]) * L[None, None, :, None] / r
    assert np.all(np.abs(got - counts) < 0.25), np.abs(got - counts).max()
    np.testing.assert_allclose(to_f64(gpu["lse"]), np.broadcast_to(np.log(L), (B, H, N)),
                               atol=1e-4)


@pytest.mark.parametrize("d,N,dtype", [(64, 200, torch.bfloat16), (128, 300, torch.float16)])
def test_backward_mask_read_out_exactly(d, N, dtype):
    """Q = 0, no causal mask: P_ij = 1 / N, so dV_jc = r / N * (kept queries i = c mod d of
    key j) when dO_i = e_(i mod d)."""
    B, H, p, seed, off = 2, 2, 0.4, 2024, 1
    t = oracle.dropout_threshold(p)
    r = 256 / (256 - t)
    q = torch.zeros((B, H, N, d), dtype=dtype)
    k = torch.randn((B, H, N, d)).to(dtype)
    v = torch.randn((B, H, N, d)).to(dtype)
    do = torch.zeros((B, H, N, d), dtype=dtype)
    do[:, :, torch.arange(N), torch.arange(N) % d] = 1
    gpu = run_dropout(q, k, v, do, scale=0.125, causal=False, kv_len=None, p=p, seed=seed,
                      offset=off)
    keep = oracle_mask(B, H, N, p, seed, off).astype(np.int64)  # [B,H,i,j]
    counts = np.zeros((B, H, N, d), np.int64)                     # [B,H,j,c]
    for c in range(d):
        counts[..., c] = keep[:, :, np.arange(N) % d == c, :].sum(axis=2)
    got = to_f64(gpu["dv"]) * N / r
    assert np.all(np.abs(got - counts) < 0.25), np.abs(got - counts).max()


CASES = [
    # (B, H, N, d, dtype, causal, kv_range, p, seed)
    (2, 2, 200, 64, torch.bfloat16, True, None, 0.1, 1),
    (2, 3, 300, 128, torch.float16, False, (100, 300), 0.3, 2),
    (1, 2, 517, 64, torch.float16, False, (1, 517), 0.5, 3),
    (1, 2, 640, 128, torch.bfloat16, True, None, 0.2, 4),
    (2, 2, 1024, 64, torch.bfloat16, True, None, 0.1, 5),
    (1, 1, 1, 64, torch.bfloat16, False, None, 0.5, 6),
    (3, 1, 129, 128, torch.bfloat16, False, None, 0.9, 7),
]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kvr,p,seed", CASES)
def test_dropout_matches_oracle(B, H, N, d, dtype, causal, kvr, p, seed):
    w = W.custom(B=B, H=H, N=N, d=d, dtype=dtype, causal=causal, kv_len_range=kvr)
    inp = W.make_inputs(w, seed=seed)
    off = seed * 11
    gpu = run_dropout(inp["q"], inp["k"], inp["v"], inp["do"], scale=w.scale, causal=causal,
                      kv_len=inp["kv_len"], p=p, seed=seed, offset=off)
    kv = None if inp["kv_len"] is None else inp["kv_len"].numpy()
    ref = oracle.attention(*(to_f64(inp[n]) for n in ("q", "k", "v", "do")), scale=w.scale,
                           causal=causal, kv_len=kv, dropout_p=p, seed=seed, offset=off)
    f = compare_forward(gpu, ref, out_scale=keep_scale(p))
    g = compare_backward(gpu, ref)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert max(g.values()) <= GRAD_REL_L2, g


def test_zero_probability_matches_dense_path():
    w = W.custom(B=2, H=2, N=300, d=64, dtype=torch.bfloat16, causal=True)
    inp = W.make_inputs(w, seed=12)
    drop = run_dropout(inp["q"], inp["k"], inp["v"], inp["do"], scale=w.scale, causal=True,
                       kv_len=None, p=0.0, seed=1, offset=0)
    from parity import run_gpu
    dense = run_gpu(inp, w.scale, True)
    # at d = 64 the dense path has its own kernel (split rows, 3/8 of the exponentials from
    # a polynomial with relative error <= 7.5e-5): the same LSE up to that error in the
    # normaliser and fp32 summation order
    assert torch.allclose(drop["lse"], dense["lse"], atol=2e-4, rtol=0), \
        (drop["lse"] - dense["lse"]).abs().max()
    for n in ("o", "dq", "dk", "dv"):
        a, b = drop[n].float(), dense[n].float()
        assert torch.allclose(a, b, atol=2e-2, rtol=2e-2), (n, (a - b).abs().max())


def test_different_seeds_and_offsets_differ_and_repeat():
    w = W.custom(B=1, H=2, N=256, d=64, dtype=torch.bfloat16)
    inp = W.make_inputs(w, seed=3)
    args = dict(scale=w.scale, causal=False, kv_len=None, p=0.5, backward=False)
    a = run_dropout(inp["q"], inp["k"], inp["v"], None, seed=1, offset=0, **args)
    b = run_dropout(inp["q"], inp["k"], inp["v"], None, seed=1, offset=0, **args)
    c = run_dropout(inp["q"], inp["k"], inp["v"], None, seed=2, offset=0, **args)
    e = run_dropout(inp["q"], inp["k"], inp["v"], None, seed=1, offset=1, **args)
    assert torch.equal(a["o"], b["o"])
    assert not torch.equal(a["o"], c["o"]) and not torch.equal(a["o"], e["o"])


def test_gpt2_shape_sampled_rows():
    """GPT-2 shape (B8 H12 N1024 d64 bf16 causal) with p = 0.1: every output of three
    heads against the oracle."""
    w = W.WORKLOADS["gpt2"]
    inp = W.make_inputs(w, seed=0)
    p, seed, off = 0.1, 42, 0
    gpu = run_dropout(inp["q"], inp["k"], inp["v"], inp["do"], scale=w.scale, causal=True,
                      kv_len=None, p=p, seed=seed, offset=off)
    heads = [(0, 0), (3, 7), (7, 11)]
    ref = oracle.attention(*(to_f64(inp[n]) for n in ("q", "k", "v", "do")), scale=w.scale,
                           causal=True, heads=heads, dropout_p=p, seed=seed, offset=off)
    mask = np.zeros((w.B, w.H), bool)
    for b, h in heads:
        mask[b, h] = True
    f = compare_forward(gpu, ref, mask, out_scale=keep_scale(p))
    g = compare_backward(gpu, ref, mask)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert max(g.values()) <= GRAD_REL_L2, g
