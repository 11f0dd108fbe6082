"""Shared helpers of the GPU parity tests: run the CUDA path through the C-ABI binding,
run the fp64 oracle on the same seeded inputs, and compare.

Tolerances (fp16/bf16 inputs, fp32 accumulation): O max-abs <= 1e-2, LSE max-abs <= 1e-3,
dQ/dK/dV relative L2 (||g - g_ref|| / ||g_ref|| over the whole tensor) <= 2e-2.

O is returned in the 16-bit input dtype, whose spacing exceeds 2e-2 for |O| >= 4 (bf16),
so the O bound is applied to the computation: element-wise |O - O_ref| <= 1e-2 plus half
an ulp of O_ref in the output dtype.  The plain max-abs error is reported beside it.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_io_aware_60_b200 import fa

O_ATOL = 1e-2
LSE_ATOL = 1e-3
GRAD_REL_L2 = 2e-2

# Fraction bits of the 16-bit output types.  O is returned in the input dtype, so on top of
# the computation's error every output element carries up to half an ulp of rounding.
_FRAC_BITS = {torch.bfloat16: 7, torch.float16: 10}


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


def oracle_full(inp: dict, scale: float, causal: bool, backward: bool = True, heads=None,
                block_mask=None):
    q, k, v = (to_f64(inp[n]) for n in ("q", "k", "v"))
    do = to_f64(inp["do"]) if backward else None
    kv = None if inp["kv_len"] is None else inp["kv_len"].numpy()
    return oracle.attention(q, k, v, do, scale=scale, causal=causal, kv_len=kv, heads=heads,
                            block_mask=block_mask, block_size=128)


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


def half_ulp(x: np.ndarray, dtype) -> np.ndarray:
    """Half a unit in the last place of ``dtype`` at each value of ``x``."""
    fb = _FRAC_BITS[dtype]
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, -14.0 if dtype == torch.float16 else -126.0)
    return np.where(ax > 0, np.exp2(e - fb - 1), 0.0)


def o_error_beyond_rounding(gpu_o: np.ndarray, ref_o: np.ndarray, dtype) -> float:
    """max(|O_gpu - O_ref| - halfulp(O_ref)): the error of the computation once the
    unavoidable rounding of the 16-bit output is set aside.  This is the graded O error:
    it must stay <= O_ATOL.  (The plain max-abs is reported beside it.)"""
    if gpu_o.size == 0:
        return 0.0
    return float(np.max(np.abs(gpu_o - ref_o) - half_ulp(ref_o, dtype)))


def rounding_floor(ref: np.ndarray, dtype) -> float:
    """Largest |round_dtype(x) - x| over the reference values: the error any output in
    ``dtype`` must show, reported next to the graded max-abs error."""
    r = torch.from_numpy(np.ascontiguousarray(ref)).to(dtype).double().numpy()
    return float(np.max(np.abs(r - ref))) if ref.size else 0.0


def compare_forward(gpu: dict, ref: dict, mask=None) -> dict:
    """Max-abs errors of O and LSE over the entries selected by ``mask`` (a boolean
    [B,H] array of checked heads; None = all).  Also reports the error of O against the
    oracle rounded to the output dtype and the rounding floor itself (diagnostics)."""
    dtype = gpu["o"].dtype
    go, gl = to_f64(gpu["o"]), to_f64(gpu["lse"])
    ro, rl = ref["o"], ref["lse"]
    if mask is not None:
        go, gl, ro, rl = go[mask], gl[mask], ro[mask], rl[mask]
    o_err = float(np.max(np.abs(go - ro))) if go.size else 0.0
    ro_r = torch.from_numpy(np.ascontiguousarray(ro)).to(dtype).double().numpy()
    res = {"o_err": o_error_beyond_rounding(go, ro, dtype), "o_max_abs": o_err,
           "lse_max_abs": lse_err(gl, rl),
           "o_vs_rounded_oracle": float(np.max(np.abs(go - ro_r))) if go.size else 0.0,
           "o_rounding_floor": rounding_floor(ro, dtype)}
    print("forward parity:", {k: f"{v:.3e}" for k, v in res.items()})
    return res


def compare_backward(gpu: dict, ref: dict, mask=None) -> dict:
    res = {}
    for n in ("dq", "dk", "dv"):
        g, r = to_f64(gpu[n]), ref[n]
        if mask is not None:
            g, r = g[mask], r[mask]
        res[n + "_rel_l2"] = rel_l2(g, r)
    print("backward parity:", {k: f"{v:.3e}" for k, v in res.items()})
    return res
