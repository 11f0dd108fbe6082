"""Pins of the oracle for queries and keys of different lengths (the inference shape:
a short block of new queries against a long key sequence; stackzen.ai glossary entry
"FlashAttention", which cites the method's saving at inference).  The Nq queries are the last Nq positions of the Nk-long sequence, so
causal masking keeps key j for query i when j <= i + Nk - Nq.

Fixed from outside the oracle by: brute-force softmax without the max shift on tiny
rectangular inputs; the identity that a rectangular problem equals the last Nq rows of the
square problem over the whole sequence; the closed form of a single query with Q = 0;
central finite differences."""
import numpy as np
import pytest

import oracle


def brute(q, k, v, scale, causal, L):
    Nq, Nk = q.shape[0], k.shape[0]
    S = scale * (q @ k.T)
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    allowed = (j < L) & ((not causal) | (j <= i + Nk - Nq))
    E = np.where(allowed, np.exp(np.where(allowed, S, 0.0)), 0.0)
    Z = E.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        P = np.where(Z[:, None] > 0, E / Z[:, None], 0.0)
        lse = np.where(Z > 0, np.log(Z), -np.inf)
    return P @ v, lse


@pytest.mark.parametrize("Nq,Nk,causal,L", [(1, 7, False, 7), (1, 7, True, 5), (3, 8, True, 8),
                                            (2, 9, False, 4), (5, 5, True, 5), (4, 6, True, 3),
                                            (6, 3, False, 3)])
def test_brute_force_rectangular(Nq, Nk, causal, L):
    r = np.random.default_rng(Nq * 10 + Nk)
    q = r.standard_normal((Nq, 4))
    k, v = r.standard_normal((Nk, 4)), r.standard_normal((Nk, 4))
    res = oracle.attention_rows(q, k, v, scale=0.6, causal=causal, kv_len=L)
    o, lse = brute(q, k, v, 0.6, causal, L)
    np.testing.assert_allclose(res["o"], o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(res["lse"], lse, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L", [40, 25])
def test_last_rows_of_the_square_problem(causal, L):
    """Queries Nk-Nq .. Nk-1 of a square problem see exactly what the rectangular problem
    with those Nq queries sees."""
    r = np.random.default_rng(3)
    Nk, Nq, d = 40, 6, 8
    q, k, v, do = (r.standard_normal((Nk, d)) for _ in range(4))
    sq = oracle.attention_rows(q, k, v, do, scale=0.4, causal=causal, kv_len=L,
                               rows=np.arange(Nk - Nq, Nk))
    rect = oracle.attention_rows(q[Nk - Nq:], k, v, do[Nk - Nq:], scale=0.4, causal=causal,
                                 kv_len=L)
    for name in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(rect[name], sq[name], rtol=1e-12, atol=1e-13, err_msg=name)


def test_single_query_zero_is_mean_of_valid_values():
    r = np.random.default_rng(4)
    k, v = r.standard_normal((50, 3)), r.standard_normal((50, 3))
    res = oracle.attention_rows(np.zeros((1, 3)), k, v, scale=1.0, causal=True, kv_len=31)
    np.testing.assert_allclose(res["o"][0], v[:31].mean(axis=0), atol=1e-14)
    np.testing.assert_allclose(res["lse"][0], np.log(31.0), atol=1e-14)


def test_rectangular_gradients_finite_differences():
    r = np.random.default_rng(5)
    Nq, Nk, d = 3, 7, 3
    q, do = r.standard_normal((Nq, d)), r.standard_normal((Nq, d))
    k, v = r.standard_normal((Nk, d)), r.standard_normal((Nk, d))
    kw = dict(scale=0.7, causal=True, kv_len=6)
    res = oracle.attention_rows(q, k, v, do, **kw)

    def loss():
        return float((oracle.attention_rows(q, k, v, **kw)["o"] * do).sum())
    eps = 1e-6
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        g = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            old = x[idx]
            x[idx] = old + eps
            a = loss()
            x[idx] = old - eps
            b = loss()
            x[idx] = old
            g[idx] = (a - b) / (2 * eps)
        assert np.linalg.norm(res[name] - g) / np.linalg.norm(g) < 1e-6, name


def test_rectangular_rejects_block_mask_and_dropout():
    r = np.random.default_rng(6)
    q, k = r.standard_normal((2, 4)), r.standard_normal((5, 4))
    with pytest.raises(RuntimeError):
        oracle.attention_rows(q, k, k, scale=1.0, block_mask=np.ones((1, 1)), block_size=128)
    with pytest.raises(RuntimeError):
        oracle.attention_rows(q, k, k, scale=1.0, dropout_p=0.5, seed=1)
