#!/usr/bin/env python
"""Benchmark of the exact-attention hot path (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one forward pass and one backward pass of the whole path over one batch of
the GPT-2-small shaped workload (B8 H12 N1024 d64 bf16, causal), seeded synthetic data.
The metric is attention forward+backward TFLOP/s with the nominal FLOP count
(4 B H N^2 d forward, 2.5x that backward, halved for causal).  Prints ONE JSON line.

Multi-GPU (one process per GPU under torchrun): every rank runs its own batch (weak
scaling); the heads are independent, so there is no data-path collective; the timed
region is bracketed by barriers and the reported time is the maximum over ranks.

``--impl reference`` times the fp64 CPU oracle (test infrastructure) on the host cores,
each step one bounded sample of the same workload; only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s (bf16, 1×B200) and % of dense tensor-core peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "gpt2"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
REASON_FIELDS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


# ------------------------------------------------------------------ host-side helpers
# (kept free of CUDA so that the multi-rank logic is testable with gloo on CPU)

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch (weak scaling)."""
    return 1000 * rank


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def quantise_e4m3(x):
    """Per-tensor E4M3 quantisation of a host tensor: (bytes, scale factor)."""
    import torch
    s = float(x.float().abs().max()) / 448.0
    return (x.float() / s).to(torch.float8_e4m3fn), s


def step_flops(w, block_mask=None, fwd_only=False) -> tuple:
    """(forward, backward, total) FLOPs of one step.  Dense: the nominal count.  With a
    block mask: 4 d per visible (query, key) pair forward and 10 d backward (the work the
    kernels actually do; masked blocks are skipped).  Inference shape or FP8: forward
    only."""
    if w.inference or fwd_only:
        f = w.nominal_flops()[0]
        return f, 0.0, f
    if block_mask is None:
        f, b = w.nominal_flops()
        return f, b, f + b
    vis = visible_pairs(w.N, block_mask, w.causal)
    f = 4.0 * w.d * vis * w.B * w.H
    return f, 2.5 * f, 3.5 * f


def local_global_mask(T: int):
    """Block pattern of the block-sparse measurement: every query tile sees its own and the
    previous key tile (local band) and the first key tile (global)."""
    import numpy as np
    m = np.zeros((T, T), dtype=np.uint8)
    for i in range(T):
        m[i, max(0, i - 1):i + 1] = 1
        m[i, 0] = 1
    return m


def visible_pairs(N: int, mask, causal: bool) -> int:
    """Number of (query, key) pairs the mask (128 x 128 blocks) and the causal rule allow."""
    T = mask.shape[0]
    total = 0
    for qt in range(T):
        rows = min(128, N - qt * 128)
        for kt in range(T):
            if not mask[qt, kt]:
                continue
            cols = min(128, N - kt * 128)
            if not causal or kt < qt:
                total += rows * cols
            elif kt == qt:
                total += sum(min(r + 1, cols) for r in range(rows))
    return total


def whole_job_tflops(flops_per_step: float, n_gpus: int, steps: int, max_ms: float) -> float:
    return n_gpus * flops_per_step * steps / (max_ms * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# The sources a kernel's profile depends on: its own header, the shared helpers, and the
# host function in fa_api.cu that configures and launches it.
KERNEL_SOURCES = {
    "fa_fwd_kernel": (("fa_fwd.cuh", "sm100.cuh", "dropout.cuh"),
                      ("launch_fwd", "make_map", "launch_pdl", "set_smem", "balance_items",
                       "schedule_for", "no_schedule")),
    "fa_bwd_kernel": (("fa_bwd.cuh", "sm100.cuh", "dropout.cuh"),
                      ("launch_bwd", "bwd_workspace_layout", "make_map", "launch_pdl",
                       "set_smem", "grid_for", "balance_items", "schedule_for", "no_schedule")),
}


def _code_only(src: str) -> str:
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return " ".join(src.split())


def _function_text(src: str, name: str) -> str:
    """The text of the top-level host function ``name`` in ``src``: from the line that
    starts its definition (return type at the start of the line, the name followed by
    ``(``, not a call or a declaration ending in ``;``) to its closing brace at the start
    of a line.  Empty if there is no such definition."""
    for m in re.finditer(rf"(?m)^[A-Za-z_][\w:<>, \t\*&]*\b{re.escape(name)}\(", src):
        start = m.start()
        brace = src.find("{", m.end())
        semi = src.find(";", m.end())
        if brace < 0 or (0 <= semi < brace):
            continue  # a declaration
        end = src.find("\n}\n", start)
        return src[start:end + 3 if end >= 0 else len(src)]
    return ""


def kernel_source_sha(kernel: str = None) -> str:
    """Hash of CUDA code with comments removed and whitespace collapsed, so that a profile
    summary stays valid across comment and layout edits and goes stale on any change to
    the code.  With ``kernel`` (a key of KERNEL_SOURCES): only the files and the launch
    function that kernel depends on; without: every source (for the launch list)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_60_b200", "csrc")
    if kernel is None:
        names = sorted(n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh")))
        for n in names:
            with open(os.path.join(csrc, n), encoding="utf-8") as f:
                h.update(_code_only(f.read()).encode())
        return h.hexdigest()[:16]
    files, functions = KERNEL_SOURCES[kernel]
    for n in files:
        path = os.path.join(csrc, n)
        if os.path.exists(path):
            with open(path, encoding="utf-8") as f:
                h.update(_code_only(f.read()).encode())
    api = os.path.join(csrc, "fa_api.cu")
    if os.path.exists(api):
        with open(api, encoding="utf-8") as f:
            src = f.read()
        for fn in functions:
            h.update(_code_only(_function_text(src, fn)).encode())
    return h.hexdigest()[:16]


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of ``kernel`` from the committed ncu summary, if that summary
    was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    try:
        with open(path) as f:
            txt = f.read()
    except OSError:
        return None
    vals = {}
    for line in txt.splitlines():
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha") != kernel_source_sha(kernel):
        return None
    try:
        # (a scaled capture states its factor after the number)
        return float(vals["dram_bytes_per_launch"].split()[0])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons of one GPU in the background."""

    QUERY = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[3], parts[5:9]))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= self.t1]
        note = "samples inside the timed region"
        if not inside:
            inside = rows
            note = "timed region shorter than the sampling period: samples of the whole run"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "no samples"}
        reasons = set()
        for r in inside:
            for name, val in zip(REASON_FIELDS, r[4]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside), "note": note}


def gpu_pci_id(dev: int) -> str:
    import torch
    p = torch.cuda.get_device_properties(dev)
    try:
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except AttributeError:
        return str(dev)


# ------------------------------------------------------------------ our arm

def inference_bytes(w) -> float:
    """Compulsory HBM bytes of one inference forward: read Q, K, V, write O and LSE."""
    e = 2
    return float(w.B * w.H * (2 * w.N * w.d * e + 2 * w.n_q * w.d * e + 4 * w.n_q))


def alloc_set(w, inp, dev, fp8=False):
    import torch
    from exact_io_aware_60_b200 import fa
    if fp8:
        s = {}
        for n in ("q", "k", "v"):
            x8, sc = quantise_e4m3(inp[n])
            s[n] = x8.to(dev)
            s[n + "_scale"] = sc
        s["kv_len"] = None if inp["kv_len"] is None else inp["kv_len"].to(dev)
        s["o"] = torch.empty(s["q"].shape, dtype=torch.bfloat16, device=dev)
        s["lse"] = torch.empty(s["q"].shape[:-1], dtype=torch.float32, device=dev)
        s["fp8"] = True
        return s
    if w.inference:
        s = {n: inp[n].to(dev) for n in ("q", "k", "v")}
        s["kv_len"] = None if inp["kv_len"] is None else inp["kv_len"].to(dev)
        s["o"] = torch.empty_like(s["q"])
        s["lse"] = torch.empty(s["q"].shape[:-1], dtype=torch.float32, device=dev)
        n = fa.fa_fwd_splitkv_workspace_bytes(w.B, w.H, w.n_q, w.N, w.d, 0)
        s["ws_split"] = torch.empty(n, dtype=torch.uint8, device=dev) if n > 0 else None
        return s
    s = {n: inp[n].to(dev) for n in ("q", "k", "v", "do")}
    s["kv_len"] = None if inp["kv_len"] is None else inp["kv_len"].to(dev)
    s["o"] = torch.empty_like(s["q"])
    s["lse"] = torch.empty(s["q"].shape[:-1], dtype=torch.float32, device=dev)
    s["dq"], s["dk"], s["dv"] = (torch.empty_like(s["q"]) for _ in range(3))
    s["ws"] = fa.workspace_for(s["q"])
    return s


def set_bytes(s) -> int:
    import torch
    return sum(t.numel() * t.element_size() for n, t in s.items() if isinstance(t, torch.Tensor))


def run_step(w, s, stream=None):
    from exact_io_aware_60_b200 import fa
    if s.get("fp8"):
        fa.fa_fwd_fp8(s["q"], s["k"], s["v"], s["o"], s["lse"], scale=w.scale,
                      q_scale=s["q_scale"], k_scale=s["k_scale"], v_scale=s["v_scale"],
                      causal=w.causal, kv_len=s["kv_len"], stream=stream)
        return
    if w.inference:
        fa.fa_fwd_splitkv(s["q"], s["k"], s["v"], s["o"], s["lse"], scale=w.scale,
                          causal=w.causal, kv_len=s["kv_len"], num_splits=0,
                          workspace=s["ws_split"], stream=stream)
        return
    if s.get("drop") is not None:
        p, seed = s["drop"]
        fa.fa_fwd_dropout(s["q"], s["k"], s["v"], s["o"], s["lse"], scale=w.scale, p_drop=p,
                          seed=seed, causal=w.causal, kv_len=s["kv_len"], stream=stream)
        fa.fa_bwd_dropout(s["q"], s["k"], s["v"], s["o"], s["do"], s["lse"], s["dq"], s["dk"],
                          s["dv"], scale=w.scale, p_drop=p, seed=seed, causal=w.causal,
                          kv_len=s["kv_len"], workspace=s["ws"], stream=stream)
        return
    if s.get("mask") is not None:
        fa.fa_fwd_blocksparse(s["q"], s["k"], s["v"], s["o"], s["lse"], s["mask"], scale=w.scale,
                              causal=w.causal, kv_len=s["kv_len"], stream=stream)
        fa.fa_bwd_blocksparse(s["q"], s["k"], s["v"], s["o"], s["do"], s["lse"], s["dq"],
                              s["dk"], s["dv"], s["mask"], scale=w.scale, causal=w.causal,
                              kv_len=s["kv_len"], workspace=s["ws"], stream=stream)
        return
    fa.fa_fwd(s["q"], s["k"], s["v"], s["o"], s["lse"], scale=w.scale, causal=w.causal,
              kv_len=s["kv_len"], stream=stream)
    fa.fa_bwd(s["q"], s["k"], s["v"], s["o"], s["do"], s["lse"], s["dq"], s["dk"], s["dv"],
              scale=w.scale, causal=w.causal, kv_len=s["kv_len"], workspace=s["ws"],
              stream=stream)


def cpu_baseline_sample(w, inp, budget_s: float, dropout_p: float = 0.0, fp8_set=None) -> dict:
    """The oracle (as it stands) on whole heads of the workload until ``budget_s`` of CPU
    time has passed (at least one head)."""
    import oracle
    if fp8_set is not None:  # the values the E4M3 inputs represent
        q, k, v = (fp8_set[n].cpu().double().numpy() * fp8_set[n + "_scale"]
                   for n in ("q", "k", "v"))
        do = None
    else:
        q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
        do = None if w.inference else inp["do"].double().numpy()
    kv = None if inp["kv_len"] is None else inp["kv_len"].numpy()
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    t0 = time.perf_counter()
    done = 0
    for b, h in heads:
        L = w.N if kv is None else int(kv[b])
        oracle.attention_rows(q[b, h], k[b, h], v[b, h], None if do is None else do[b, h],
                              scale=w.scale,
                              causal=w.causal, kv_len=L, dropout_p=dropout_p, seed=1234,
                              bh=b * w.H + h)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    flops = step_flops(w, fwd_only=do is None)[2] * done / (w.B * w.H)
    cores = oracle.threads()
    # the same oracle on one core, one (batch, head) pair
    one = None
    if do is not None and w.N <= 4096:
        b, h = heads[0]
        L = w.N if kv is None else int(kv[b])
        oracle.set_threads(1)
        t1 = time.perf_counter()
        oracle.attention_rows(q[b, h], k[b, h], v[b, h], do[b, h], scale=w.scale,
                              causal=w.causal, kv_len=L, dropout_p=dropout_p, seed=1234, bh=b * w.H + h)
        one_dt = time.perf_counter() - t1
        oracle.set_threads(cores)
        one = {"value": step_flops(w)[2] / (w.B * w.H) / one_dt / 1e12, "unit": UNIT, "cores": 1,
               "sample": f"one (batch, head) pair in {one_dt:.3f} s"}
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cores,
            "kind": "oracle", "one_core": one,
            "sample": f"fp64 oracle {'forward' if do is None else 'forward+backward'} of "
                      f"{done} of {w.B * w.H} (batch, head) "
                      f"pairs of the {w.name} workload"
                      + (f" with dropout p={dropout_p}" if dropout_p else "")
                      + f" in {dt:.1f} s (nominal FLOPs)"}


def config_dict(w, args, world: int) -> dict:
    """The workload description both arms print (identical for the same flags)."""
    mask = local_global_mask((w.N + 127) // 128) if args.block_sparse else None
    return {"workload": w.description
            + (", E4M3 inputs (per-tensor scales), forward only" if args.fp8 else
               ", inference forward (split-KV)" if w.inference else ", forward + backward")
            + (", block-sparse local+global pattern" if args.block_sparse else "")
            + (f", dropout p={args.dropout}" if args.dropout > 0 else ""),
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            **({"Nq": w.n_q} if w.inference else {}),
            "flops_per_step": step_flops(w, mask, fwd_only=args.fp8)[2],
            "parallelism": f"replicas x{world} (no collective)",
            "l2": "inputs rotated over resident sets totalling more than twice the 126 MB L2, "
                  "so each step reads data evicted from it"}


def kernel_sample_pass(w, sets, nsets, stream, dev, steps):
    """``steps`` steps with CUDA events recorded by the library around the forward kernel
    and the backward main kernel (on the launch stream).  Returns {0: [(start, stop)],
    1: [...]}; the caller reads the elapsed times."""
    import torch
    from exact_io_aware_60_b200 import fa
    evs = {0: [], 1: []}
    for which in (0, 1):
        for _ in range(steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            b.record(stream)
            evs[which].append((a, b))
    torch.cuda.synchronize(dev)
    for i in range(steps):
        fa.fa_set_timing_events(0, *evs[0][i])
        fa.fa_set_timing_events(1, *evs[1][i])
        run_step(w, sets[i % nsets])
    fa.fa_set_timing_events(0)
    fa.fa_set_timing_events(1)
    torch.cuda.synchronize(dev)
    return evs


# Other workloads measured after the headline one (forward + backward each): the kernels'
# TFLOP/s and fraction of the tensor peak, and for the key-padded BERT shape, which sits at
# the ridge point, the forward's achieved HBM bandwidth and its effective FLOPs as well.
OTHER_WORKLOADS = ("bert", "long16k", "causal64k")


def fwd_compulsory_bytes(w) -> float:
    """HBM bytes a forward pass must move: read Q, K, V, write O (16-bit) and LSE (fp32)."""
    return float(w.B * w.H * w.N * (4 * w.d * 2 + 4))


def effective_flops(w, kv_len) -> tuple:
    """(forward, backward) FLOPs over the pairs the key-padding mask leaves visible (the
    kernels skip padded key blocks): 4 d per visible (query, key) pair forward, 10 d
    backward."""
    if kv_len is None:
        return w.nominal_flops()
    L = [min(w.N, max(0, int(x))) for x in kv_len]
    pairs = 0.0
    for Lb in L:
        pairs += sum(min(Lb, i + 1) for i in range(w.N)) if w.causal else float(w.N) * Lb
    f = 4.0 * w.d * w.H * pairs
    return f, 2.5 * f


def measure_other_workload(name, dev, stream, steps, peak, hbm, args):
    import torch
    from exact_io_aware_60_b200 import workloads as W
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=0)
    first = alloc_set(w, inp, dev)
    per_set = set_bytes(first)
    nsets = 1 if per_set > 2 * 126 * 2 ** 20 else 2
    sets = [first] + [alloc_set(w, W.make_inputs(w, seed=i), dev) for i in range(1, nsets)]
    for i in range(3):
        run_step(w, sets[i % nsets])
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        run_step(w, sets[i % nsets])
    b.record(stream)
    torch.cuda.synchronize(dev)
    step_ms = a.elapsed_time(b) / steps
    evs = kernel_sample_pass(w, sets, nsets, stream, dev, steps)
    f_fwd, f_bwd = w.nominal_flops()
    k_f = sum(x.elapsed_time(y) for x, y in evs[0]) / steps
    k_b = sum(x.elapsed_time(y) for x, y in evs[1]) / steps
    tf = lambda f, ms: f / (ms * 1e-3) / 1e12
    fk, bk = "fa_fwd_kernel", "fa_bwd_kernel"
    res = {"workload": w.description, "steps": steps, "inputs_sets": nsets,
           "ms_per_step": step_ms, "tflops_step": tf(f_fwd + f_bwd, step_ms),
           fk: {"ms": k_f, "tflops": tf(f_fwd, k_f), "frac": tf(f_fwd, k_f) / peak},
           bk: {"ms": k_b, "tflops": tf(f_bwd, k_b), "frac": tf(f_bwd, k_b) / peak}}
    if inp["kv_len"] is not None:
        e_fwd, e_bwd = effective_flops(w, inp["kv_len"].tolist())
        gbs = fwd_compulsory_bytes(w) / (k_f * 1e-3) / 1e9
        res[fk].update({
            "effective_tflops": tf(e_fwd, k_f), "effective_frac": tf(e_fwd, k_f) / peak,
            "hbm_bytes": fwd_compulsory_bytes(w), "hbm_gbs": gbs, "hbm_frac": gbs / hbm})
        res[bk].update({"effective_tflops": tf(e_bwd, k_b),
                        "effective_frac": tf(e_bwd, k_b) / peak})
    del sets, first
    torch.cuda.empty_cache()
    return res


def bench_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from exact_io_aware_60_b200 import fa
    from exact_io_aware_60_b200 import workloads as W

    if world > 1 and not dist.is_initialized():
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = W.WORKLOADS[args.workload]
    if args.heads > 0:
        w = dataclasses.replace(w, H=args.heads,
                                description=w.description + f" (reduced to H={args.heads})")
    mask_np = local_global_mask((w.N + 127) // 128) if args.block_sparse else None
    f_fwd, f_bwd, f_step = step_flops(w, mask_np, fwd_only=args.fp8)

    inp = W.make_inputs(w, seed=rank_seed(rank), with_grad=not args.fp8)
    first = alloc_set(w, inp, dev, fp8=args.fp8)
    per_set = set_bytes(first)
    l2 = 126 * 2 ** 20
    nsets = max(2, math.ceil(2 * l2 / per_set) + 1)
    sets = [first] + [alloc_set(w, W.make_inputs(w, seed=rank_seed(rank) + i,
                                                 with_grad=not args.fp8), dev, fp8=args.fp8)
                      for i in range(1, nsets)]
    if mask_np is not None:
        mask_t = torch.from_numpy(mask_np).to(dev)
        for st in sets:
            st["mask"] = mask_t
    if args.dropout > 0:
        for i, st in enumerate(sets):
            st["drop"] = (args.dropout, 1234 + i)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for i in range(args.warmup):
        run_step(w, sets[i % nsets])
    torch.cuda.synchronize(dev)
    status = fa.fa_get_device_status()
    if status != fa.FA_OK:
        raise RuntimeError(f"device status {status} after warm-up")

    # The headline region: K steps back to back, no per-kernel events (an event between two
    # kernels keeps the next one from starting early under programmatic dependent launch).
    K = args.steps
    fa.fa_set_timing_events(0)
    fa.fa_set_timing_events(1)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(gpu_pci_id(local_rank))
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.mark("t0")
    start.record(stream)
    for i in range(K):
        run_step(w, sets[i % nsets])
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark("t1")
    barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    status = fa.fa_get_device_status()
    if status != fa.FA_OK:
        raise RuntimeError(f"device status {status} after the timed region")
    ms = start.elapsed_time(end)
    max_ms = max_over_ranks(ms, dev if world > 1 else None)
    value = whole_job_tflops(f_step, world, K, max_ms)

    # Per-kernel device times (forward kernel, backward main kernel) from a separate pass of
    # the same steps on the same rotated inputs, with events around those two launches.
    evs = kernel_sample_pass(w, sets, nsets, stream, dev, max(3, min(K, args.kernel_steps)))
    fwd_only = w.inference or args.fp8
    k_fwd = sum(a.elapsed_time(b) for a, b in evs[0]) / len(evs[0])
    k_bwd = 0.0 if fwd_only else sum(a.elapsed_time(b) for a, b in evs[1]) / len(evs[1])

    def spread(pairs):
        ts = sorted(a.elapsed_time(b) for a, b in pairs)
        pick = lambda q: ts[min(len(ts) - 1, int(q * (len(ts) - 1) + 0.5))]
        return {"calls": len(ts), "median_ms": pick(0.5), "p10_ms": pick(0.1), "p90_ms": pick(0.9)}
    fwd_name, bwd_name = "fa_fwd_kernel", "fa_bwd_kernel"
    per_call = {fwd_name: spread(evs[0])}
    if not fwd_only:
        per_call[bwd_name] = spread(evs[1])

    # back-to-back steps on one input set (inputs warm in the 126 MB L2), labelled as such
    Kw = min(K, 200)
    wa, wb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wa.record(stream)
    for _ in range(Kw):
        run_step(w, first)
    wb.record(stream)
    torch.cuda.synchronize(dev)
    warm_ms = wa.elapsed_time(wb)
    warm = {"ms_per_step": warm_ms / Kw, "value": f_step / (warm_ms / Kw * 1e-3) / 1e12,
            "unit": UNIT, "steps": Kw, "note": "one input set reused: warm L2, not the headline"}
    peak_mem = int(torch.cuda.max_memory_allocated(dev))

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        in_names = ("q", "k", "v") if fwd_only else ("q", "k", "v", "do")
        out_names = ("o", "lse") if fwd_only else ("o", "lse", "dq", "dk", "dv")
        if args.fp8:
            host = {n: first[n].cpu().pin_memory() for n in in_names}
        else:
            host = {n: inp[n].pin_memory() for n in in_names}
        outs = {n: torch.empty(first[n].shape, dtype=first[n].dtype, pin_memory=True)
                for n in out_names}
        Ke = max(3, min(K, args.e2e_steps))
        s = first

        def e2e_step():
            for n in in_names:
                s[n].copy_(host[n], non_blocking=True)
            run_step(w, s)
            for n in out_names:
                outs[n].copy_(s[n], non_blocking=True)

        def timed(fn):
            for i in range(2):
                fn(i)
            torch.cuda.synchronize(dev)
            barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(Ke):
                fn(i)
            end_fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            return max_over_ranks(a.elapsed_time(b), dev if world > 1 else None)

        # serial: copy in, step, copy out, one after the other on one stream
        end_fn = lambda: None
        serial_ms = timed(lambda i: e2e_step())

        # pipelined: two device sets; the inputs of step i+1 go up on one copy stream and
        # the outputs of step i-1 come down on another while step i computes
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_pipelined(i):
            kk = i % 2
            st = sets[kk]
            h2d.wait_stream(stream) if i == 0 else h2d.wait_event(ev_done[kk])
            with torch.cuda.stream(h2d):
                for n in in_names:
                    st[n].copy_(host[n], non_blocking=True)
                ev_in[kk].record(h2d)
            stream.wait_event(ev_in[kk])
            if i >= 2:
                stream.wait_event(ev_out[kk])  # outputs of step i-2 have left this set
            run_step(w, st, stream=stream)
            ev_done[kk].record(stream)
            d2h.wait_event(ev_done[kk])
            with torch.cuda.stream(d2h):
                for n in out_names:
                    outs[n].copy_(st[n], non_blocking=True)
                ev_out[kk].record(d2h)

        def end_pipelined():
            stream.wait_stream(d2h)
            stream.wait_stream(h2d)

        end_fn = end_pipelined
        e_ms = timed(e2e_pipelined)
        e2e = {"value": whole_job_tflops(f_step, world, Ke, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host.values()),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs.values()),
               "steps": Ke, "ms_per_step": e_ms / Ke,
               "note": "copies of step i+1 (in) and i-1 (out) overlap step i: two device "
                       "buffer sets, one copy stream each way",
               "serial": {"value": whole_job_tflops(f_step, world, Ke, serial_ms),
                          "ms_per_step": serial_ms / Ke}}

    peaks, peak_src = load_peaks()
    sustained = ms > 1000.0
    peak_key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    if args.fp8:
        peak *= 2.0  # E4M3 dense peak: the measured bf16 figure x the nominal ratio 4.5 / 2.25
    # the dominant kernel is the one with the larger device time per step
    if k_bwd >= k_fwd:
        dom_name, dom_flops, dom_ms = bwd_name, f_bwd, k_bwd
    else:
        dom_name, dom_flops, dom_ms = fwd_name, f_fwd, k_fwd
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": dom_name, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{peak_src} {peak_key}"
                               + (" x 2 (e4m3 / bf16 nominal)" if args.fp8 else ""),
                "flops_per_launch": dom_flops, "launch_ms": dom_ms,
                "launches_timed": len(evs[0]),
                "timing": "CUDA events around each launch in a sampled pass after the "
                          "headline region",
                "traffic": profile_traffic(dom_name, w.name)}
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    if w.inference and f_fwd / inference_bytes(w) < peak * 1e3 / hbm:
        # below the ridge point: the split-KV forward is bound by streaming K and V
        gbs = inference_bytes(w) / (dom_ms * 1e-3) / 1e9
        roofline.update({"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "peak_source": f"{peak_src} hbm_gbs",
                         "bytes_per_launch": inference_bytes(w), "tflops": achieved})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(w, inp, args.cpu_seconds, args.dropout,
                                  fp8_set=first if args.fp8 else None)

    others = None
    if (args.workload == DEFAULT_WORKLOAD and not (args.block_sparse or args.dropout or args.fp8)
            and not args.no_other_workloads):
        others = {}
        for name in OTHER_WORKLOADS:
            others[name] = measure_other_workload(name, dev, stream, args.other_steps, peak, hbm,
                                                  args)
        status = fa.fa_get_device_status()
        if status != fa.FA_OK:
            raise RuntimeError(f"device status {status} after the other workloads")

    per_rank_value = f_step * K / (ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": max_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if args.fp8 else {torch.bfloat16: "bf16", torch.float16: "f16"}[w.dtype],
        "data": "synthetic (seeded N(0,1), GPT-2-small shapes; no dataset)",
        "config": config_dict(w, args, world),
        "l2_sets": f"{nsets} resident input/output sets ({nsets * per_set / 2**20:.0f} MiB)",
        "pct_of_peak": 100.0 * per_rank_value / peak,
        "kernels": ({fwd_name: {"ms": k_fwd, "tflops": f_fwd / (k_fwd * 1e-3) / 1e12,
                                "frac": f_fwd / (k_fwd * 1e-3) / 1e12 / peak}}
                    if fwd_only else
                    {fwd_name: {"ms": k_fwd, "tflops": f_fwd / (k_fwd * 1e-3) / 1e12,
                                "frac": f_fwd / (k_fwd * 1e-3) / 1e12 / peak},
                     bwd_name: {"ms": k_bwd, "tflops": f_bwd / (k_bwd * 1e-3) / 1e12,
                                       "frac": f_bwd / (k_bwd * 1e-3) / 1e12 / peak}}),
        "roofline": roofline,
        "per_call": per_call,
        "kernel_times": "per-kernel figures from a separate pass of the same steps with "
                        "events around the two kernels; the headline region has none",
        "warm_l2": warm,
        "peak_mem_bytes": peak_mem,
        "e2e": e2e,
        "gpu_launches": (K if args.fp8 else
                         (1 + int(first.get("ws_split") is not None)) * K if w.inference
                         else 4 * K),
        "clocks": clk,
        "cpu_baseline": cpu,
        "other_workloads": others,
    }
    if world > 1:
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()
    return line


# ------------------------------------------------------------------ reference arm

def bench_reference(args):
    """The fp64 oracle on the host cores; each step is one bounded sample of the workload
    (the forward + backward of one (batch, head) pair, or of a row subset of it when the
    requested step count would not finish within a few minutes)."""
    import numpy as np
    import oracle
    from exact_io_aware_60_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    inp = W.make_inputs(w, seed=0, with_grad=not args.fp8)
    if args.fp8:  # the values the E4M3 inputs represent
        q, k, v = (x8.double().numpy() * sc for x8, sc in
                   (quantise_e4m3(inp[n]) for n in ("q", "k", "v")))
        do = None
    else:
        q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
        do = None if w.inference else inp["do"].double().numpy()
    kv = None if inp["kv_len"] is None else inp["kv_len"].numpy()
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    total = args.steps + args.warmup
    nq = w.n_q
    rows_per_step = nq if total <= 300 else max(min(16, nq), (nq * 300) // total)
    # about 2^22 score rows x keys per step at most, so a step stays a fraction of a second
    rows_per_step = min(rows_per_step, max(16, (1 << 22) // w.N))
    rng = np.random.default_rng(0)
    off = w.N - nq  # inference shape: queries are the last nq positions

    bmask = local_global_mask((w.N + 127) // 128) if args.block_sparse else None

    def flops_of(rows, L):
        vis = 0
        for i in rows:
            lim = min(L, i + 1 + off) if w.causal else L  # keys < lim pass causal/padding
            if bmask is None:
                vis += lim
            else:
                for kt in np.nonzero(bmask[i // 128])[0]:
                    vis += max(0, min(lim, (kt + 1) * 128) - kt * 128)
        # 4d forward (+ 10d backward) per visible score
        return (4.0 if do is None else 14.0) * w.d * vis

    def one(i):
        b, h = heads[i % len(heads)]
        L = w.N if kv is None else int(kv[b])
        rows = (np.arange(nq) if rows_per_step >= nq
                else np.sort(rng.choice(nq, rows_per_step, replace=False)))
        oracle.attention_rows(q[b, h], k[b, h], v[b, h], None if do is None else do[b, h],
                              scale=w.scale,
                              causal=w.causal, kv_len=L, rows=rows, dropout_p=args.dropout,
                              seed=1234, bh=b * w.H + h, block_mask=bmask, block_size=128)
        return flops_of(rows, L)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    fl = 0.0
    for i in range(args.steps):
        fl += one(args.warmup + i)
    dt = time.perf_counter() - t0
    value = fl / dt / 1e12
    sample = (f"fp64 oracle {'forward' if do is None else 'forward+backward'} of "
              f"{rows_per_step} query rows of one (batch, head) pair per step, {w.name} workload")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), GPT-2-small shapes; no dataset)",
        "config": config_dict(w, args, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-steps", type=int, default=64,
                    help="steps of the per-kernel timing pass after the headline region")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the BERT / long16k / causal64k kernel measurements")
    ap.add_argument("--other-steps", type=int, default=5)
    ap.add_argument("--heads", type=int, default=0,
                    help="profiling: run the workload with this many heads instead of its own "
                         "(a smaller launch of the same kernel shape for counter captures)")
    ap.add_argument("--block-sparse", action="store_true",
                    help="measure the block-sparse path with a local+global block pattern "
                         "(FLOPs counted over the visible pairs only)")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="measure the dropout path with this drop probability")
    ap.add_argument("--fp8", action="store_true",
                    help="measure the E4M3 forward (d = 128 workloads; forward only)")
    args = ap.parse_args(argv)
    if args.fp8 and (args.dropout or args.block_sparse):
        ap.error("--fp8 measures the plain E4M3 forward")
    if args.dropout and args.block_sparse:
        ap.error("--dropout and --block-sparse measure different paths; pick one")
    if not (0.0 <= args.dropout < 255.5 / 256):
        ap.error("--dropout must lie in [0, 255.5/256)")
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(bench_reference(args)), flush=True)
        return 0
    line = bench_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
