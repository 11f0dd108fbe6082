"""Seeded synthetic inputs shaped like the workloads the FlashAttention pages measure.

This module holds no attention arithmetic: it only draws random tensors.  The CUDA
path's tests, the oracle's tests and ``bench.py`` all take their inputs from here, so
both sides see bit-identical values.

Recipe (for every workload): ``torch.Generator('cpu').manual_seed(seed)``; draw fp32
``randn`` of shape ``[B, H, N, d]`` in the order Q, K, V, dO; then, where the workload
has them, the per-sequence key lengths (``randint(lo, hi + 1, (B,))``) and the seeded
key permutation whose first ``floor(frac * N)`` positions get their key vectors scaled.
Scaling factors are powers of two, so scaling before or after the cast gives the same
values.  Everything is finally cast to the workload's dtype on the host.

The five named workloads stand in for the pages' benchmarks (promptingindex page
"FlashAttention: The IO-Aware Algorithm That Rewrote GPU Training Speed Records",
section "Benchmark results"): GPT-2 at sequence 1K, BERT-large at sequence 512,
Path-X at 16K and Path-256 at 64K.  Only their shapes are used; no dataset item is.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: torch.dtype
    causal: bool = False
    kv_len_range: Optional[tuple] = None   # (lo, hi) inclusive, per sequence
    input_scale: float = 1.0               # multiplies Q, K, V (a power of two)
    spike_frac: float = 0.0                # fraction of key positions scaled
    spike_scale: float = 1.0               # factor for those keys (a power of two)
    description: str = ""
    # Inference shape: Nq queries against N keys (the queries are the last Nq positions of
    # the sequence); None = training shape with Nq = N.
    Nq: Optional[int] = None

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def n_q(self) -> int:
        return self.N if self.Nq is None else self.Nq

    @property
    def inference(self) -> bool:
        return self.Nq is not None

    def nominal_flops(self) -> tuple:
        """(forward, backward) FLOPs: 4 B H N^2 d forward, 2.5x backward, halved causal.
        Inference shape: 4 d per visible (query, key) pair, i.e. Nq N pairs, less
        Nq (Nq - 1) / 2 under causal masking (bottom-right aligned)."""
        if self.inference:
            pairs = self.n_q * self.N
            if self.causal:
                pairs -= self.n_q * (self.n_q - 1) / 2
            f = 4.0 * self.B * self.H * self.d * pairs
            return f, 2.5 * f
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        if self.causal:
            f *= 0.5
        return f, 2.5 * f


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 128, 64, torch.float16,
                     description="B1 H2 N128 d64 fp16, no mask"),
    "gpt2": Workload("gpt2", 8, 12, 1024, 64, torch.bfloat16, causal=True,
                     description="GPT-2-small shaped: B8 H12 N1024 d64 bf16 causal"),
    "bert": Workload("bert", 16, 16, 512, 64, torch.float16, kv_len_range=(256, 512),
                     description="BERT-large shaped: B16 H16 N512 d64 fp16, key padding "
                                 "lengths uniform in [256, 512]"),
    "long16k": Workload("long16k", 1, 8, 16384, 64, torch.bfloat16, input_scale=0.5,
                        description="long context: B1 H8 N16384 d64 bf16, Q/K/V x0.5"),
    "causal64k": Workload("causal64k", 1, 16, 65536, 128, torch.bfloat16, causal=True,
                          spike_frac=0.01, spike_scale=8.0,
                          description="very long causal: B1 H16 N65536 d128 bf16, 1% of "
                                      "keys x8"),
    # inference shapes (forward only): new queries against a long key sequence
    "decode32k": Workload("decode32k", 8, 16, 32768, 128, torch.bfloat16, causal=True, Nq=1,
                          description="inference decode: B8 H16, 1 query against 32768 keys, "
                                      "d128 bf16"),
    "chunk16k": Workload("chunk16k", 1, 16, 16384, 128, torch.bfloat16, causal=True, Nq=512,
                         description="inference prefill chunk: B1 H16, 512 queries against "
                                     "16384 keys, d128 bf16 causal"),
}


def custom(name="custom", *, B, H, N, d, dtype=torch.bfloat16, causal=False,
           kv_len_range=None, input_scale=1.0, spike_frac=0.0, spike_scale=1.0) -> Workload:
    return Workload(name, B, H, N, d, dtype, causal, kv_len_range, input_scale,
                    spike_frac, spike_scale)


def make_inputs(w: Workload, seed: int = 0, with_grad: bool = True) -> dict:
    """Host (CPU) tensors for workload ``w``: q, k, v, do in ``w.dtype`` (``[B,H,N,d]``,
    contiguous; q and do ``[B,H,Nq,d]`` for an inference shape), ``kv_len`` (int32 ``[B]``
    or None), ``spike_keys`` (int64 or None)."""
    g = torch.Generator("cpu").manual_seed(seed)
    shape = (w.B, w.H, w.N, w.d)
    qshape = (w.B, w.H, w.n_q, w.d)
    q = torch.randn(qshape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(qshape, generator=g, dtype=torch.float32) if with_grad else None
    kv_len = None
    if w.kv_len_range is not None:
        lo, hi = w.kv_len_range
        kv_len = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64)
        kv_len = kv_len.to(torch.int32)
    spike = None
    if w.spike_frac > 0.0:
        cnt = int(math.floor(w.spike_frac * w.N))
        spike = torch.randperm(w.N, generator=g)[:cnt].sort().values
    if w.input_scale != 1.0:
        q.mul_(w.input_scale)
        k.mul_(w.input_scale)
        v.mul_(w.input_scale)
    if spike is not None:
        k[:, :, spike, :] *= w.spike_scale
    out = {
        "q": q.to(w.dtype).contiguous(),
        "k": k.to(w.dtype).contiguous(),
        "v": v.to(w.dtype).contiguous(),
        "do": None if do is None else do.to(w.dtype).contiguous(),
        "kv_len": kv_len,
        "spike_keys": spike,
    }
    return out
