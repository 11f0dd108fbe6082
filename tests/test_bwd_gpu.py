"""GPU backward parity: dQ, dK, dV from the CUDA path (through the C ABI) against the fp64
oracle on identical seeded inputs; relative L2 error <= 2e-2 per gradient tensor.  The
forward outputs that feed the backward pass come from the CUDA forward."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_60_b200 import fa
from exact_io_aware_60_b200 import workloads as W
from parity import (GRAD_REL_L2, LSE_ATOL, O_ATOL, compare_backward, compare_forward,
                    o_graded_error, oracle_full, rel_l2, rounding_floor, run_gpu,
                    to_f64)

pytestmark = pytest.mark.gpu

EDGE = [
    # (N, d, dtype, causal, kv_len_range)
    (1, 64, torch.bfloat16, False, None),
    (2, 128, torch.float16, True, None),
    (17, 64, torch.float16, True, None),
    (127, 128, torch.bfloat16, False, None),
    (128, 64, torch.bfloat16, True, None),
    (129, 64, torch.float16, False, None),
    (200, 128, torch.bfloat16, True, (60, 200)),
    (255, 64, torch.bfloat16, False, (1, 255)),
    (384, 64, torch.float16, True, (0, 384)),
    (517, 128, torch.float16, False, None),
    (640, 64, torch.bfloat16, True, None),
]


@pytest.mark.parametrize("N,d,dtype,causal,kvr", EDGE)
def test_backward_edge_shapes(N, d, dtype, causal, kvr):
    w = W.custom(B=2, H=3, N=N, d=d, dtype=dtype, causal=causal, kv_len_range=kvr)
    inp = W.make_inputs(w, seed=1000 + N + d)
    gpu = run_gpu(inp, w.scale, causal)
    ref = oracle_full(inp, w.scale, causal)
    f = compare_forward(gpu, ref)
    g = compare_backward(gpu, ref)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert max(g.values()) <= GRAD_REL_L2, g
    if kvr is not None:
        # keys past the valid length get exact-zero gradients
        for b in range(w.B):
            L = int(inp["kv_len"][b])
            assert torch.all(gpu["dk"][b, :, L:] == 0) and torch.all(gpu["dv"][b, :, L:] == 0)


# d = 64 at 4096 rows and more (32+ query tiles per head): ragged tails, causal masking,
# key padding (including an empty sequence).
LONG_EDGE = [
    # (N, dtype, causal, kv_len_range)
    (4096, torch.bfloat16, True, None),
    (4173, torch.float16, False, None),
    (4224, torch.bfloat16, True, (0, 4224)),
    (4353, torch.bfloat16, False, (1, 4353)),
]


@pytest.mark.parametrize("N,dtype,causal,kvr", LONG_EDGE)
def test_backward_long_d64_edge_shapes(N, dtype, causal, kvr):
    w = W.custom(B=2, H=1, N=N, d=64, dtype=dtype, causal=causal, kv_len_range=kvr)
    inp = W.make_inputs(w, seed=2000 + N)
    gpu = run_gpu(inp, w.scale, causal)
    ref = oracle_full(inp, w.scale, causal)
    f = compare_forward(gpu, ref)
    g = compare_backward(gpu, ref)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert max(g.values()) <= GRAD_REL_L2, g
    if kvr is not None:
        for b in range(w.B):
            L = int(inp["kv_len"][b])
            assert torch.all(gpu["dk"][b, :, L:] == 0) and torch.all(gpu["dv"][b, :, L:] == 0)


def test_backward_zero_length_sequence():
    w = W.custom(B=2, H=2, N=160, d=64, dtype=torch.bfloat16)
    inp = W.make_inputs(w, seed=11)
    inp["kv_len"] = torch.tensor([0, 97], dtype=torch.int32)
    gpu = run_gpu(inp, w.scale, False)
    for n in ("dq", "dk", "dv"):
        assert torch.all(gpu[n][0] == 0), n
    ref = oracle_full(inp, w.scale, False)
    g = compare_backward(gpu, ref)
    assert max(g.values()) <= GRAD_REL_L2, g


@pytest.mark.parametrize("name", ["tiny", "gpt2", "bert"])
def test_backward_named_workloads_full(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=0)
    gpu = run_gpu(inp, w.scale, w.causal)
    ref = oracle_full(inp, w.scale, w.causal)
    f = compare_forward(gpu, ref)
    g = compare_backward(gpu, ref)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert max(g.values()) <= GRAD_REL_L2, g


def test_backward_long16k_two_full_heads():
    """Full-size launch (B1 H8 N16384 d64); the oracle evaluates two seeded heads in full
    (every row of dQ, dK, dV); the other heads are checked by the gradient identities."""
    w = W.WORKLOADS["long16k"]
    inp = W.make_inputs(w, seed=0)
    gpu = run_gpu(inp, w.scale, w.causal)
    heads = [(0, 2), (0, 7)]
    ref = oracle_full(inp, w.scale, w.causal, heads=heads)
    mask = np.zeros((w.B, w.H), dtype=bool)
    for b, h in heads:
        mask[b, h] = True
    f = compare_forward(gpu, ref, mask)
    g = compare_backward(gpu, ref, mask)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert max(g.values()) <= GRAD_REL_L2, g
    check_identities(gpu, inp, w)


def check_identities(gpu, inp, w):
    """Rows of P sum to one and rows of dS sum to zero, so for every head
    sum_j dV_j = sum_i dO_i and sum_j dK_j = 0 (up to bf16 rounding of the outputs)."""
    dv = gpu["dv"].double().sum(dim=2)
    do = inp["do"].double().sum(dim=2)
    dk = gpu["dk"].double().sum(dim=2)
    scale_dv = gpu["dv"].double().abs().sum(dim=2)
    scale_dk = gpu["dk"].double().abs().sum(dim=2)
    assert torch.all((dv - do).abs() <= 2e-2 * scale_dv + 1e-3)
    assert torch.all(dk.abs() <= 2e-2 * scale_dk + 1e-3)


def test_backward_causal64k_sampled():
    """Full-size launch (B1 H16 N65536 d128 causal, 1% keys x8).  The oracle checks, for two
    seeded heads: sampled dQ rows (each from its own full score row), and dK/dV of the last
    1024 keys, which only the last 1024 query rows can see under the causal mask, so the
    oracle over those rows gives their exact gradients.  All heads: gradient identities."""
    w = W.WORKLOADS["causal64k"]
    inp = W.make_inputs(w, seed=0)
    gpu = run_gpu(inp, w.scale, w.causal)
    check_identities(gpu, inp, w)
    rng = np.random.default_rng(5)
    N = w.N
    tail = 1024
    for b, h in [(0, 4), (0, 13)]:
        q, k, v, do = (to_f64(inp[n][b, h]) for n in ("q", "k", "v", "do"))
        rows = np.unique(np.concatenate([np.arange(N - tail, N),
                                         rng.choice(N - tail, size=48, replace=False),
                                         np.array([0, 1, 127, 128])]))
        ref = oracle.attention_rows(q, k, v, do, scale=w.scale, causal=True, rows=rows)
        gdq = to_f64(gpu["dq"][b, h])[rows]
        go = to_f64(gpu["o"][b, h])[rows]
        errs = {"dq_rel_l2": rel_l2(gdq, ref["dq"]),
                "o_err": o_graded_error(go, ref["o"], w.dtype),
                "o_max_abs": float(np.max(np.abs(go - ref["o"]))),
                "o_rounding_floor": rounding_floor(ref["o"], w.dtype)}
        # keys >= N - tail are seen only by rows >= N - tail, all of which are in `rows`
        for n in ("dk", "dv"):
            g = to_f64(gpu[n][b, h])[N - tail:]
            errs[n + "_rel_l2"] = rel_l2(g, ref[n][N - tail:])
        print(f"causal64k head {(b, h)}:", {k: f"{v:.3e}" for k, v in errs.items()})
        assert errs["o_err"] <= O_ATOL, errs
        assert max(errs[n] for n in ("dq_rel_l2", "dk_rel_l2", "dv_rel_l2")) <= GRAD_REL_L2, errs


def test_backward_is_deterministic_in_dk_dv():
    """dK and dV are accumulated inside one CTA in a fixed order: two runs agree bitwise.
    (dQ is summed across CTAs with atomics and may differ in the last bits.)"""
    w = W.WORKLOADS["gpt2"]
    inp = W.make_inputs(w, seed=3)
    a = run_gpu(inp, w.scale, w.causal)
    b = run_gpu(inp, w.scale, w.causal)
    assert torch.equal(a["dk"], b["dk"]) and torch.equal(a["dv"], b["dv"])
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"])
