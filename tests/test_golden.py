"""The stored oracle snapshot (tests/golden/oracle_small.json) still reproduces, and a
brute-force softmax without max shift agrees with it (forward values)."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_small.json")


def cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", cases(), ids=lambda c: c["name"])
def test_oracle_reproduces_snapshot(case):
    arr = {n: np.array(case[n]) for n in ("q", "k", "v", "do")}
    res = oracle.attention_rows(arr["q"], arr["k"], arr["v"], arr["do"], scale=case["scale"],
                                causal=case["causal"], kv_len=case["kv_len"])
    for n in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(res[n], np.array(case[n]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("case", cases(), ids=lambda c: c["name"])
def test_snapshot_forward_matches_brute_force(case):
    q, k, v = (np.array(case[n]) for n in ("q", "k", "v"))
    N = q.shape[0]
    S = case["scale"] * q @ k.T
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    ok = (j < case["kv_len"]) & ((not case["causal"]) | (j <= i))
    E = np.where(ok, np.exp(S), 0.0)
    np.testing.assert_allclose(np.array(case["o"]), (E / E.sum(1, keepdims=True)) @ v, atol=1e-13)
    np.testing.assert_allclose(np.array(case["lse"]), np.log(E.sum(1)), atol=1e-13)
