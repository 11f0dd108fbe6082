"""Writes ``oracle_small.json``: the fp64 oracle's outputs on two small fixed inputs.

Only ``oracle/`` computes the stored values.  The inputs are small dyadic numbers
(exactly representable in fp16, bf16 and fp64) so that the same fixture also serves
as a fixed GPU parity case.  The stored values are a regression snapshot of the
oracle; ``tests/test_golden.py`` also re-derives them with a brute-force softmax.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def dyadic(shape, seed):
    r = np.random.default_rng(seed)
    return r.integers(-8, 9, size=shape) / 8.0


def main():
    cases = []
    for name, N, d, causal, L, seed in (("noncausal_N6_d4_L5", 6, 4, False, 5, 1),
                                        ("causal_N7_d2", 7, 2, True, 7, 2)):
        q, k, v, do = (dyadic((N, d), seed * 10 + t) for t in range(4))
        scale = 0.5
        res = oracle.attention_rows(q, k, v, do, scale=scale, causal=causal, kv_len=L)
        cases.append({
            "name": name, "N": N, "d": d, "causal": causal, "kv_len": L, "scale": scale,
            "q": q.tolist(), "k": k.tolist(), "v": v.tolist(), "do": do.tolist(),
            "o": res["o"].tolist(), "lse": res["lse"].tolist(), "dq": res["dq"].tolist(),
            "dk": res["dk"].tolist(), "dv": res["dv"].tolist(),
        })
    doc = {
        "about": "fp64 oracle outputs (standard attention, its definition: anthology note "
                 "'NOTE-005: FlashAttention', Theorem 1) on fixed dyadic inputs; written by "
                 "tests/golden/make_golden.py, which calls only oracle/",
        "cases": cases,
    }
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(out, "w") as f:
        json.dump(doc, f, indent=1)
    print("wrote", out)


if __name__ == "__main__":
    main()
