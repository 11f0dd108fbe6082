"""The seeded input generator: determinism, shapes, dtypes and the workload recipes."""
import math

import torch

from exact_io_aware_60_b200 import workloads as W


def test_named_workloads_shapes():
    assert (W.WORKLOADS["gpt2"].B, W.WORKLOADS["gpt2"].H, W.WORKLOADS["gpt2"].N,
            W.WORKLOADS["gpt2"].d) == (8, 12, 1024, 64)
    assert W.WORKLOADS["causal64k"].d == 128 and W.WORKLOADS["causal64k"].causal
    f, b = W.WORKLOADS["gpt2"].nominal_flops()
    assert f == 0.5 * 4 * 8 * 12 * 1024 ** 2 * 64 and b == 2.5 * f


def test_deterministic_and_dtype():
    w = W.WORKLOADS["tiny"]
    a, b = W.make_inputs(w, seed=0), W.make_inputs(w, seed=0)
    for n in ("q", "k", "v", "do"):
        assert a[n].dtype == torch.float16 and a[n].shape == (1, 2, 128, 64)
        assert torch.equal(a[n], b[n])
    c = W.make_inputs(w, seed=1)
    assert not torch.equal(a["q"], c["q"])


def test_kv_len_range_and_order():
    w = W.custom(B=64, H=1, N=8, d=4, kv_len_range=(3, 6))
    x = W.make_inputs(w, seed=3)
    assert x["kv_len"].dtype == torch.int32
    assert int(x["kv_len"].min()) >= 3 and int(x["kv_len"].max()) <= 6
    # Q, K, V, dO are drawn before kv_len: the tensors equal those of the unpadded recipe.
    y = W.make_inputs(W.custom(B=64, H=1, N=8, d=4), seed=3)
    assert torch.equal(x["q"], y["q"]) and torch.equal(x["do"], y["do"])


def test_spiked_keys_and_input_scale():
    w = W.custom(B=1, H=2, N=400, d=8, spike_frac=0.01, spike_scale=8.0, input_scale=0.5,
                 dtype=torch.float32)
    x = W.make_inputs(w, seed=4)
    y = W.make_inputs(W.custom(B=1, H=2, N=400, d=8, dtype=torch.float32), seed=4)
    spike = x["spike_keys"]
    assert spike.numel() == math.floor(0.01 * 400)
    mask = torch.zeros(400, dtype=torch.bool)
    mask[spike] = True
    assert torch.equal(x["k"][:, :, mask], y["k"][:, :, mask] * 4.0)
    assert torch.equal(x["k"][:, :, ~mask], y["k"][:, :, ~mask] * 0.5)
    assert torch.equal(x["q"], y["q"] * 0.5)
