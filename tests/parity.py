"""Shared helpers of the GPU parity tests: run the CUDA path through the C-ABI binding,
run the fp64 oracle on the same seeded inputs, and compare.

Tolerances (fp16/bf16 inputs, fp32 accumulation): O max-abs <= 1e-2, LSE max-abs <= 1e-3,
dQ/dK/dV relative L2 (||g - g_ref|| / ||g_ref|| over the whole tensor) <= 2e-2.

O is returned in the 16-bit input dtype.  Where |O_ref| >= 4 in bf16 the spacing is 2^-5,
so rounding the exact value alone can be off by 2^-6 = 0.0156 > 1e-2 and no bf16 output
can meet the bound there.  Element-wise, the graded rule is therefore
    |O - O_ref| <= max(1e-2, halfulp(O_ref) + 2e-3),
which is the plain 1e-2 bound wherever half an ulp plus the small computation allowance
fits under it (|O| < 4 in bf16, every fp16 value below 8), and half an ulp plus 2e-3 only
where it does not.  The plain max-abs error is reported beside the graded one.

Gradients are also graded per (batch, head): a head's error norm over the larger of its
own reference norm and the root-mean-square head norm stays <= 2e-2, so an error confined
to part of one head cannot hide in the norm over all heads.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_io_aware_60_b200 import fa

O_ATOL = 1e-2
# Allowance for the computation on top of half an ulp of output rounding, used only where
# that sum exceeds O_ATOL (large |O|; see the module docstring).
O_EPS = 2e-3
LSE_ATOL = 1e-3
GRAD_REL_L2 = 2e-2
GRAD_REL_L2_HEAD = 2e-2

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


def o_graded_error(gpu_o: np.ndarray, ref_o: np.ndarray, dtype, out_scale: float = 1.0) -> float:
    """The graded O error, which must stay <= O_ATOL: max over elements of
    |O_gpu - O_ref| - max(0, halfulp(O_ref) + O_EPS - O_ATOL).  An element passes exactly
    when |O_gpu - O_ref| <= max(O_ATOL, halfulp(O_ref) + O_EPS); where half an ulp plus
    O_EPS fits under O_ATOL the grade is the plain error.

    ``out_scale`` s > 1 is for outputs that are s times a convex combination of rows of V
    (attention dropout, s = 1 / (1 - p)): their computation error scales with s, so the
    bounds apply to O / s, i.e. |O_gpu - O_ref| <= max(s O_ATOL, halfulp(O_ref) + s O_EPS),
    reported in units of O / s."""
    if gpu_o.size == 0:
        return 0.0
    s = float(out_scale)
    excess = np.maximum(0.0, half_ulp(ref_o, dtype) + s * O_EPS - s * O_ATOL)
    return float(np.max(np.abs(gpu_o - ref_o) - excess)) / s


def rounding_floor(ref: np.ndarray, dtype) -> float:
    """Largest |round_dtype(x) - x| over the reference values: the error any output in
    ``dtype`` must show, reported next to the graded max-abs error."""
    r = torch.from_numpy(np.ascontiguousarray(ref)).to(dtype).double().numpy()
    return float(np.max(np.abs(r - ref))) if ref.size else 0.0


def compare_forward(gpu: dict, ref: dict, mask=None, out_scale: float = 1.0) -> dict:
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
    res = {"o_err": o_graded_error(go, ro, dtype, out_scale), "o_max_abs": o_err,
           "lse_max_abs": lse_err(gl, rl),
           "o_vs_rounded_oracle": float(np.max(np.abs(go - ro_r))) if go.size else 0.0,
           "o_rounding_floor": rounding_floor(ro, dtype)}
    print("forward parity:", {k: f"{v:.3e}" for k, v in res.items()})
    return res


def head_rel_l2_max(g: np.ndarray, r: np.ndarray) -> float:
    """Largest per-head error norm, each over max(that head's reference norm, the
    root-mean-square head norm).  ``g``, ``r``: [heads, rows, d] (or [B, H, rows, d]).
    The floor keeps heads whose exact gradient is zero (e.g. a sequence with one visible
    key) from dividing rounding noise by zero."""
    g = g.reshape(-1, *g.shape[-2:])
    r = r.reshape(-1, *r.shape[-2:])
    if g.shape[0] == 0:
        return 0.0
    num = np.sqrt(np.sum((g - r) ** 2, axis=(1, 2)))
    den = np.sqrt(np.sum(r ** 2, axis=(1, 2)))
    floor = np.sqrt(np.sum(den ** 2) / den.size)
    if floor == 0.0:
        return float(np.max(num))
    return float(np.max(num / np.maximum(den, floor)))


def compare_backward(gpu: dict, ref: dict, mask=None) -> dict:
    """Relative L2 error of dQ, dK, dV over the selected heads (the graded figure,
    <= GRAD_REL_L2) and the largest per-head figure (<= GRAD_REL_L2_HEAD, the same
    bound).  Returns both kinds of keys; every value must stay within 2e-2."""
    res = {}
    for n in ("dq", "dk", "dv"):
        g, r = to_f64(gpu[n]), ref[n]
        if mask is not None:
            g, r = g[mask], r[mask]
        res[n + "_rel_l2"] = rel_l2(g, r)
        res[n + "_head_max"] = head_rel_l2_max(g, r)
    assert GRAD_REL_L2_HEAD == GRAD_REL_L2  # callers grade max(values) against one bound
    print("backward parity:", {k: f"{v:.3e}" for k, v in res.items()})
    return res
