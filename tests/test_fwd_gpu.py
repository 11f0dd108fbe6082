"""GPU forward parity: the CUDA path (through the C ABI) against the fp64 oracle on
identical seeded inputs.  O max-abs <= 1e-2 and LSE max-abs <= 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_60_b200 import workloads as W
from parity import (LSE_ATOL, O_ATOL, compare_forward, o_graded_error,
                    oracle_full, rounding_floor, run_gpu, to_f64)

pytestmark = pytest.mark.gpu

EDGE = [
    # (N, d, dtype, causal, kv_len_range)
    (1, 64, torch.bfloat16, False, None),
    (1, 128, torch.float16, True, None),
    (2, 64, torch.float16, True, None),
    (3, 128, torch.bfloat16, False, None),
    (17, 64, torch.bfloat16, True, None),
    (127, 64, torch.float16, False, None),
    (128, 128, torch.bfloat16, True, None),
    (129, 64, torch.bfloat16, True, None),
    (129, 128, torch.float16, False, None),
    (255, 64, torch.float16, False, (1, 255)),
    (300, 128, torch.bfloat16, True, (100, 300)),
    (384, 64, torch.bfloat16, False, (0, 384)),
    (517, 64, torch.bfloat16, True, None),
    (640, 128, torch.float16, True, (200, 640)),
]


@pytest.mark.parametrize("N,d,dtype,causal,kvr", EDGE)
def test_forward_edge_shapes(N, d, dtype, causal, kvr):
    w = W.custom(B=3, H=2, N=N, d=d, dtype=dtype, causal=causal, kv_len_range=kvr)
    inp = W.make_inputs(w, seed=N + d)
    gpu = run_gpu(inp, w.scale, causal, backward=False)
    ref = oracle_full(inp, w.scale, causal, backward=False)
    err = compare_forward(gpu, ref)
    assert err["o_err"] <= O_ATOL and err["lse_max_abs"] <= LSE_ATOL, err


def test_forward_zero_length_rows():
    """kv_len = 0 for one sequence: its rows see no key -> O = 0, LSE = -inf."""
    w = W.custom(B=2, H=2, N=200, d=64, dtype=torch.bfloat16)
    inp = W.make_inputs(w, seed=7)
    inp["kv_len"] = torch.tensor([0, 150], dtype=torch.int32)
    gpu = run_gpu(inp, w.scale, False, backward=False)
    assert torch.all(gpu["o"][0] == 0)
    assert torch.all(torch.isneginf(gpu["lse"][0]))
    ref = oracle_full(inp, w.scale, False, backward=False)
    err = compare_forward(gpu, ref)
    assert err["o_err"] <= O_ATOL and err["lse_max_abs"] <= LSE_ATOL, err


@pytest.mark.parametrize("name", ["tiny", "gpt2", "bert"])
def test_forward_named_workloads_full(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=0)
    gpu = run_gpu(inp, w.scale, w.causal, backward=False)
    ref = oracle_full(inp, w.scale, w.causal, backward=False)
    err = compare_forward(gpu, ref)
    assert err["o_err"] <= O_ATOL and err["lse_max_abs"] <= LSE_ATOL, err


def sample_rows(N, rng, extra=24):
    fixed = [0, 1, 2, 127, 128, 129, N // 2, N - 129, N - 128, N - 2, N - 1]
    rows = set(r for r in fixed if 0 <= r < N)
    rows.update(int(x) for x in rng.choice(N, size=extra, replace=False))
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name,heads", [("long16k", [(0, 0), (0, 5)]),
                                        ("causal64k", [(0, 3), (0, 12)])])
def test_forward_long_workloads_sampled_rows(name, heads):
    """Full-size launch; the oracle checks sampled query rows of two seeded heads (each
    row is computed from its own full score row), and every head is checked for finite
    O and LSE."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=0, with_grad=False)
    gpu = run_gpu(inp, w.scale, w.causal, backward=False)
    assert torch.isfinite(gpu["o"].float()).all() and torch.isfinite(gpu["lse"]).all()
    rng = np.random.default_rng(123)
    for b, h in heads:
        rows = sample_rows(w.N, rng)
        q, k, v = (to_f64(inp[n][b, h]) for n in ("q", "k", "v"))
        ref = oracle.attention_rows(q, k, v, scale=w.scale, causal=w.causal, rows=rows)
        go = to_f64(gpu["o"][b, h])[rows]
        gl = to_f64(gpu["lse"][b, h])[rows]
        o_max = float(np.max(np.abs(go - ref["o"])))
        o_err = o_graded_error(go, ref["o"], w.dtype)
        l_err = float(np.max(np.abs(gl - ref["lse"])))
        floor = rounding_floor(ref["o"], w.dtype)
        print(f"{name} head {(b, h)}: O error {o_err:.3e}, O max-abs {o_max:.3e} (output "
              f"rounding floor {floor:.3e}), LSE max-abs {l_err:.3e}")
        assert o_err <= O_ATOL and l_err <= LSE_ATOL, (b, h, o_err, o_max, l_err, floor)
    if name == "long16k":
        # every row sees all 16384 keys with small scores: LSE_i is close to ln N
        assert float(gpu["lse"].min()) > np.log(w.N) - 1.0
