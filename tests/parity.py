"""Shared helpers of the GPU parity tests: run the CUDA path through the C-ABI binding,
run the fp64 oracle on the same seeded inputs, and compare.

Tolerances (fp16/bf16 inputs, fp32 accumulation): O max-abs <= 1e-2, LSE max-abs <= 1e-3,
dQ/dK/dV relative L2 (||g - g_ref|| / ||g_ref|| over the whole tensor) <= 2e-2.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_io_aware_60_b200 import fa

O_ATOL = 1e-2
LSE_ATOL = 1e-3
GRAD_REL_L2 = 2e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def run_gpu(inp: dict, scale: float, causal: bool, backward: bool = True):
    dev = torch.device("cuda", 0)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    kv = None if inp["kv_len"] is None else inp["kv_len"].to(dev)
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal, kv_len=kv)
    out = {"o": o, "lse": lse}
    if backward:
        do = inp["do"].to(dev)
        dq, dk, dv = fa.backward(q, k, v, o, do, lse, scale=scale, causal=causal, kv_len=kv)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    status = fa.fa_get_device_status()
    assert status == fa.FA_OK, f"device status {status}"
    return {n: t.cpu() for n, t in out.items()}


def oracle_full(inp: dict, scale: float, causal: bool, backward: bool = True, heads=None):
    q, k, v = (to_f64(inp[n]) for n in ("q", "k", "v"))
    do = to_f64(inp["do"]) if backward else None
    kv = None if inp["kv_len"] is None else inp["kv_len"].numpy()
    return oracle.attention(q, k, v, do, scale=scale, causal=causal, kv_len=kv, heads=heads)


def lse_err(gpu_lse: np.ndarray, ref_lse: np.ndarray) -> float:
    both_inf = np.isneginf(gpu_lse) & np.isneginf(ref_lse)
    g = np.where(both_inf, 0.0, gpu_lse)
    r = np.where(both_inf, 0.0, ref_lse)
    d = np.abs(g - r)
    return float(np.nanmax(d)) if d.size else 0.0


def rel_l2(g: np.ndarray, r: np.ndarray) -> float:
    den = np.linalg.norm(r)
    num = np.linalg.norm(g - r)
    if den == 0.0:
        return float(num)
    return float(num / den)


def compare_forward(gpu: dict, ref: dict, mask=None) -> dict:
    """Max-abs errors of O and LSE over the entries selected by ``mask`` (a boolean
    [B,H] array of checked heads; None = all)."""
    go, gl = to_f64(gpu["o"]), to_f64(gpu["lse"])
    ro, rl = ref["o"], ref["lse"]
    if mask is not None:
        go, gl, ro, rl = go[mask], gl[mask], ro[mask], rl[mask]
    o_err = float(np.max(np.abs(go - ro))) if go.size else 0.0
    return {"o_max_abs": o_err, "lse_max_abs": lse_err(gl, rl)}


def compare_backward(gpu: dict, ref: dict, mask=None) -> dict:
    res = {}
    for n in ("dq", "dk", "dv"):
        g, r = to_f64(gpu[n]), ref[n]
        if mask is not None:
            g, r = g[mask], r[mask]
        res[n + "_rel_l2"] = rel_l2(g, r)
    return res
