"""Block-sparse attention on the GPU against the fp64 oracle with the same block mask
(key j visible to query i only where mask[i // 128][j // 128] != 0, on top of the causal
and key-padding rules).  Same tolerances as the dense path."""
import numpy as np
import pytest
import torch

from exact_io_aware_60_b200 import fa
from exact_io_aware_60_b200 import workloads as W
from parity import GRAD_REL_L2, LSE_ATOL, O_ATOL, compare_backward, compare_forward, oracle_full

pytestmark = pytest.mark.gpu


def run_sparse(inp, w, mask, causal):
    dev = torch.device("cuda", 0)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    kv = None if inp["kv_len"] is None else inp["kv_len"].to(dev)
    m = torch.from_numpy(np.ascontiguousarray(mask.astype(np.uint8))).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)
    fa.fa_fwd_blocksparse(q, k, v, o, lse, m, scale=w.scale, causal=causal, kv_len=kv)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    fa.fa_bwd_blocksparse(q, k, v, o, do, lse, dq, dk, dv, m, scale=w.scale, causal=causal,
                          kv_len=kv, workspace=fa.workspace_for(q))
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    return {"o": o.cpu(), "lse": lse.cpu(), "dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}


CASES = [
    # (B, H, N, d, dtype, causal, kv_range, per_head, density, seed)
    (2, 2, 517, 64, torch.bfloat16, True, None, False, 0.5, 1),
    (2, 3, 384, 128, torch.float16, False, (100, 384), True, 0.5, 2),
    (1, 2, 1024, 64, torch.bfloat16, False, None, True, 0.3, 3),
    (1, 2, 640, 128, torch.bfloat16, True, None, False, 0.7, 4),
    (3, 1, 256, 64, torch.float16, False, (30, 256), False, 0.6, 5),
    # d = 64 with 33 tiles per side, causal and key-padded
    (1, 1, 4173, 64, torch.bfloat16, True, None, False, 0.4, 6),
    (2, 1, 4224, 64, torch.float16, False, (1000, 4224), True, 0.3, 7),
]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kvr,per_head,density,seed", CASES)
def test_blocksparse_matches_oracle(B, H, N, d, dtype, causal, kvr, per_head, density, seed):
    w = W.custom(B=B, H=H, N=N, d=d, dtype=dtype, causal=causal, kv_len_range=kvr)
    inp = W.make_inputs(w, seed=seed)
    T = (N + 127) // 128
    rng = np.random.default_rng(seed)
    shape = (B, H, T, T) if per_head else (T, T)
    mask = (rng.random(shape) < density).astype(np.uint8)
    if not per_head:
        mask[0, :] = 0  # a whole query tile with no visible key
    gpu = run_sparse(inp, w, mask, causal)
    ref = oracle_full(inp, w.scale, causal, block_mask=mask)
    f = compare_forward(gpu, ref)
    g = compare_backward(gpu, ref)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert max(g.values()) <= GRAD_REL_L2, g
    if not per_head:
        rows = min(128, N)
        assert torch.all(gpu["o"][:, :, :rows] == 0) and torch.all(gpu["dq"][:, :, :rows] == 0)
        assert torch.all(torch.isneginf(gpu["lse"][:, :, :rows]))


def test_blocksparse_all_ones_equals_dense():
    w = W.custom(B=2, H=2, N=300, d=64, dtype=torch.bfloat16, causal=True)
    inp = W.make_inputs(w, seed=9)
    T = 3
    sparse = run_sparse(inp, w, np.ones((T, T), np.uint8), True)
    from parity import run_gpu
    dense = run_gpu(inp, w.scale, True)
    for n in ("o", "lse", "dk", "dv"):
        assert torch.equal(sparse[n], dense[n]), n
    assert torch.allclose(sparse["dq"].float(), dense["dq"].float(), atol=1e-2, rtol=1e-2)


def test_blocksparse_gpt2_local_global_pattern():
    """GPT-2 shape with a local (band of 2 tiles) + global (first tile) pattern."""
    w = W.WORKLOADS["gpt2"]
    inp = W.make_inputs(w, seed=0)
    T = 8
    mask = np.zeros((T, T), np.uint8)
    for i in range(T):
        mask[i, max(0, i - 1):i + 1] = 1
        mask[i, 0] = 1
    gpu = run_sparse(inp, w, mask, True)
    ref = oracle_full(inp, w.scale, True, block_mask=mask)
    f = compare_forward(gpu, ref)
    g = compare_backward(gpu, ref)
    assert f["o_err"] <= O_ATOL and f["lse_max_abs"] <= LSE_ATOL, f
    assert max(g.values()) <= GRAD_REL_L2, g
