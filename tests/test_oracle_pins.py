"""Pins of the fp64 CPU oracle against facts that do not come from the oracle itself.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign, index or mask comparison, a transposed operand, a missing scale) fails at least
one of them:

* brute-force softmax without the max shift (numpy) on tiny inputs;
* closed forms: a hand-derived worked example, Q = 0, constant V, causal row 0, N = 1,
  a large-score softmax with a known split, an empty key set;
* invariants: permutation of keys/values, key shift, row sums of P (read out through
  V = identity), scale folding;
* gradients against central finite differences of sum(O * dO), gradient identities;
* the row-subset interface used for sampled checks at full size.

The attention definition (anthology note "NOTE-005: FlashAttention", Theorem 1; the
promptingindex page, "Why attention is memory-bound, not compute-bound") fixes every
expected value here.
"""
import math

import numpy as np
import pytest

import oracle


def rng(seed):
    return np.random.default_rng(seed)


def brute_force(q, k, v, scale, causal, L):
    """Softmax computed straight from its definition: exp(S) / sum exp(S), no shift."""
    N = q.shape[0]
    S = scale * (q @ k.T)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    allowed = (j < L) & ((~np.asarray(causal)) | (j <= i))
    E = np.where(allowed, np.exp(np.where(allowed, S, 0.0)), 0.0)
    Z = E.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        P = np.where(Z[:, None] > 0, E / Z[:, None], 0.0)
        lse = np.where(Z > 0, np.log(Z), -np.inf)
    return P @ v, lse


CASES = [(N, d, causal, L) for N in (1, 2, 3, 5, 8) for d in (1, 2, 4)
         for causal in (False, True) for L in sorted({N, max(1, N - 2), 1})]


@pytest.mark.parametrize("N,d,causal,L", CASES)
def test_brute_force_softmax(N, d, causal, L):
    r = rng(1000 * N + 10 * d + causal)
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    scale = 0.7
    res = oracle.attention_rows(q, k, v, scale=scale, causal=causal, kv_len=L)
    o_bf, lse_bf = brute_force(q, k, v, scale, causal, L)
    np.testing.assert_allclose(res["o"], o_bf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(res["lse"], lse_bf, rtol=1e-12, atol=1e-13)


def test_hand_worked_example():
    """N=3, d=2, scale=1.  Scores are chosen so that exp(S) is integral:
    row 0: exp(S) = [2,1,1] -> P = [1/2,1/4,1/4], LSE = ln 4, O = [3/2, 5/4]
    row 1: exp(S) = [1,1,1] -> P = [1/3]*3,       LSE = ln 3, O = [5/3, 5/3]
    row 2: exp(S) = [1,3,1] -> P = [1/5,3/5,1/5], LSE = ln 5, O = [1, 7/5]
    Causal: row 0 sees key 0 only (O = v0, LSE = ln 2), row 1 sees keys 0,1 with equal
    scores (O = [1/2, 1/2], LSE = ln 2), row 2 is unchanged."""
    q = np.array([[math.log(2), 0.0], [0.0, 0.0], [0.0, math.log(3)]])
    k = np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 0.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0], [4.0, 4.0]])
    res = oracle.attention_rows(q, k, v, scale=1.0)
    np.testing.assert_allclose(res["o"], [[1.5, 1.25], [5 / 3, 5 / 3], [1.0, 1.4]], atol=1e-15)
    np.testing.assert_allclose(res["lse"], np.log([4.0, 3.0, 5.0]), atol=1e-15)
    res = oracle.attention_rows(q, k, v, scale=1.0, causal=True)
    np.testing.assert_allclose(res["o"], [[1.0, 0.0], [0.5, 0.5], [1.0, 1.4]], atol=1e-15)
    np.testing.assert_allclose(res["lse"], np.log([2.0, 2.0, 5.0]), atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L", [7, 4])
def test_q_zero_gives_mean_of_allowed_v(causal, L):
    N, d = 7, 3
    r = rng(5)
    k, v = r.standard_normal((N, d)), r.standard_normal((N, d))
    res = oracle.attention_rows(np.zeros((N, d)), k, v, scale=0.5, causal=causal, kv_len=L)
    for i in range(N):
        allowed = [j for j in range(N) if j < L and (not causal or j <= i)]
        np.testing.assert_allclose(res["o"][i], v[allowed].mean(axis=0), atol=1e-14)
        assert res["lse"][i] == pytest.approx(math.log(len(allowed)), abs=1e-14)


def test_constant_v_rows():
    N, d = 9, 4
    r = rng(6)
    q, k = r.standard_normal((N, d)), r.standard_normal((N, d))
    c = r.standard_normal(d)
    v = np.tile(c, (N, 1))
    for causal in (False, True):
        res = oracle.attention_rows(q, k, v, scale=1.3, causal=causal, kv_len=6)
        np.testing.assert_allclose(res["o"], np.tile(c, (N, 1)), atol=1e-14)


def test_causal_row_zero():
    N, d = 6, 4
    r = rng(7)
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    res = oracle.attention_rows(q, k, v, scale=0.25, causal=True)
    np.testing.assert_allclose(res["o"][0], v[0], atol=1e-15)
    assert res["lse"][0] == pytest.approx(0.25 * float(q[0] @ k[0]), abs=1e-15)


def test_single_token():
    r = rng(8)
    q, k, v, do = (r.standard_normal((1, 5)) for _ in range(4))
    res = oracle.attention_rows(q, k, v, do, scale=0.9, causal=True)
    np.testing.assert_allclose(res["o"], v, atol=1e-15)
    np.testing.assert_allclose(res["dq"], 0.0, atol=1e-15)
    np.testing.assert_allclose(res["dk"], 0.0, atol=1e-15)
    np.testing.assert_allclose(res["dv"], do, atol=1e-15)


def test_probability_rows_via_identity_v():
    """With d = N and V = I, O_i is the row P_i itself: check it sums to one, is zero
    where masked and positive where allowed."""
    N = 8
    r = rng(9)
    q, k = r.standard_normal((N, N)), r.standard_normal((N, N))
    for causal in (False, True):
        for L in (N, 5):
            P = oracle.attention_rows(q, k, np.eye(N), scale=0.3, causal=causal, kv_len=L)["o"]
            np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
            for i in range(N):
                for j in range(N):
                    ok = j < L and (not causal or j <= i)
                    assert (P[i, j] > 0) == ok


def test_key_value_permutation_invariance():
    N, d = 10, 4
    r = rng(10)
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    base = oracle.attention_rows(q, k, v, scale=0.5)
    perm = r.permutation(N)
    res = oracle.attention_rows(q, k[perm], v[perm], scale=0.5)
    np.testing.assert_allclose(res["o"], base["o"], atol=1e-14)
    np.testing.assert_allclose(res["lse"], base["lse"], atol=1e-14)
    res = oracle.attention_rows(q[perm], k, v, scale=0.5)
    np.testing.assert_allclose(res["o"], base["o"][perm], atol=1e-14)
    np.testing.assert_allclose(res["lse"], base["lse"][perm], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift(causal):
    """Adding u to every key adds scale*q_i.u to every score of row i: O is unchanged and
    LSE moves by exactly that amount."""
    N, d = 8, 4
    r = rng(11)
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    u = r.standard_normal(d)
    base = oracle.attention_rows(q, k, v, scale=0.6, causal=causal, kv_len=6)
    res = oracle.attention_rows(q, k + u, v, scale=0.6, causal=causal, kv_len=6)
    np.testing.assert_allclose(res["o"], base["o"], atol=1e-13)
    np.testing.assert_allclose(res["lse"], base["lse"] + 0.6 * (q @ u), atol=1e-13)


def test_scale_folds_into_q():
    N, d = 8, 4
    r = rng(12)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    a = oracle.attention_rows(q, k, v, do, scale=2.0, causal=True)
    b = oracle.attention_rows(2.0 * q, k, v, do, scale=1.0, causal=True)
    for name in ("o", "lse", "dv"):
        np.testing.assert_allclose(a[name], b[name], atol=1e-13)
    # dL/dq at scale 2 is 2 * dL/d(2q) at scale 1; dK is unchanged.
    np.testing.assert_allclose(a["dq"], 2.0 * b["dq"], atol=1e-13)
    np.testing.assert_allclose(a["dk"], b["dk"], atol=1e-13)


def test_large_scores_are_stable():
    """Scores near 1000 overflow exp() without the max shift.  Two keys with scores 1000
    and 1000 - ln 3 split the mass 3/4 : 1/4 and LSE = 1000 + ln(4/3)."""
    q = np.array([[1000.0]])
    k = np.array([[1.0], [1.0 - math.log(3) / 1000.0]])
    v = np.array([[1.0], [-3.0]])
    res = oracle.attention_rows(np.vstack([q, q]), k, v, scale=1.0)
    np.testing.assert_allclose(res["o"][:, 0], 0.75 * 1 + 0.25 * -3, atol=1e-10)
    np.testing.assert_allclose(res["lse"], 1000.0 + math.log(4 / 3), atol=1e-10)


def test_empty_key_set():
    N, d = 4, 3
    r = rng(13)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    res = oracle.attention_rows(q, k, v, do, scale=1.0, kv_len=0)
    assert np.all(res["o"] == 0.0)
    assert np.all(np.isneginf(res["lse"]))
    for name in ("dq", "dk", "dv"):
        assert np.all(res[name] == 0.0)


def loss(q, k, v, do, scale, causal, L):
    return float(np.sum(oracle.attention_rows(q, k, v, scale=scale, causal=causal,
                                              kv_len=L)["o"] * do))


@pytest.mark.parametrize("N,d,causal,L", [(5, 3, False, 5), (6, 2, True, 6), (7, 4, False, 4),
                                          (8, 3, True, 5), (4, 4, True, 1), (3, 1, False, 3)])
def test_gradients_vs_central_differences(N, d, causal, L):
    r = rng(100 + N)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    scale = 0.8
    res = oracle.attention_rows(q, k, v, do, scale=scale, causal=causal, kv_len=L)
    eps = 1e-6
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name[1]] = xp
            args_m[name[1]] = xm
            fd[idx] = (loss(args_p["q"], args_p["k"], args_p["v"], do, scale, causal, L)
                       - loss(args_m["q"], args_m["k"], args_m["v"], do, scale, causal, L)) / (2 * eps)
        err = np.linalg.norm(res[name] - fd) / max(np.linalg.norm(fd), 1e-30)
        assert err < 1e-7 or np.linalg.norm(res[name] - fd) < 1e-9, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_identities(causal):
    """Rows of P sum to 1, so sum_j dV_j = sum_i dO_i; rows of dS sum to 0, so
    sum_j dK_j = 0; keys past the valid length get exactly zero gradient."""
    N, d, L = 12, 4, 9
    r = rng(14)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    res = oracle.attention_rows(q, k, v, do, scale=0.5, causal=causal, kv_len=L)
    np.testing.assert_allclose(res["dv"].sum(axis=0), do.sum(axis=0), atol=1e-13)
    np.testing.assert_allclose(res["dk"].sum(axis=0), 0.0, atol=1e-13)
    assert np.all(res["dk"][L:] == 0.0) and np.all(res["dv"][L:] == 0.0)


def test_row_subsets_partition_the_full_result():
    """The sampled interface: any subset of rows gives the same rows, and dK/dV summed
    over a partition of the rows equal the full gradients."""
    N, d = 16, 4
    r = rng(15)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    full = oracle.attention_rows(q, k, v, do, scale=0.5, causal=True, kv_len=13)
    perm = r.permutation(N)
    parts = [perm[:5], perm[5:11], perm[11:]]
    dk = np.zeros((N, d))
    dv = np.zeros((N, d))
    for rows in parts:
        part = oracle.attention_rows(q, k, v, do, scale=0.5, causal=True, kv_len=13, rows=rows)
        for name in ("o", "dq"):
            np.testing.assert_allclose(part[name], full[name][rows], atol=1e-14)
        np.testing.assert_allclose(part["lse"], full["lse"][rows], atol=1e-14)
        dk += part["dk"]
        dv += part["dv"]
    np.testing.assert_allclose(dk, full["dk"], atol=1e-13)
    np.testing.assert_allclose(dv, full["dv"], atol=1e-13)


def test_batched_wrapper_matches_per_head():
    B, H, N, d = 2, 3, 6, 4
    r = rng(16)
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    kv_len = [6, 3]
    res = oracle.attention(q, k, v, do, scale=0.5, causal=False, kv_len=kv_len)
    for b in range(B):
        for h in range(H):
            one = oracle.attention_rows(q[b, h], k[b, h], v[b, h], do[b, h], scale=0.5,
                                        kv_len=kv_len[b])
            for name in ("o", "lse", "dq", "dk", "dv"):
                np.testing.assert_array_equal(res[name][b, h], one[name])


def test_rejects_bad_arguments():
    q = np.zeros((4, 2))
    with pytest.raises(RuntimeError):
        oracle.attention_rows(q, q, q, scale=1.0, kv_len=5)
    with pytest.raises(RuntimeError):
        oracle.attention_rows(q, q, q, scale=1.0, rows=np.array([4]))


# ---------------------------------------------------------------- block-sparse extension

def brute_force_masked(q, k, v, scale, causal, L, bmask, bs):
    N = q.shape[0]
    S = scale * (q @ k.T)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    allowed = (j < L) & ((~np.asarray(causal)) | (j <= i)) & (bmask[i // bs, j // bs] != 0)
    E = np.where(allowed, np.exp(np.where(allowed, S, 0.0)), 0.0)
    Z = E.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        P = np.where(Z[:, None] > 0, E / Z[:, None], 0.0)
        lse = np.where(Z > 0, np.log(Z), -np.inf)
    return P @ v, lse


@pytest.mark.parametrize("N,bs,causal,L", [(6, 2, False, 6), (7, 2, True, 7), (8, 3, False, 6),
                                           (8, 2, True, 5), (5, 1, False, 5)])
def test_block_mask_brute_force(N, bs, causal, L):
    r = rng(300 + N * bs)
    d = 3
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    nb = (N + bs - 1) // bs
    bmask = (r.random((nb, nb)) < 0.6).astype(np.uint8)
    res = oracle.attention_rows(q, k, v, scale=0.7, causal=causal, kv_len=L, block_mask=bmask,
                                block_size=bs)
    o_bf, lse_bf = brute_force_masked(q, k, v, 0.7, causal, L, bmask, bs)
    np.testing.assert_allclose(res["o"], o_bf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(res["lse"], lse_bf, rtol=1e-12, atol=1e-13)


def test_block_mask_all_ones_is_dense():
    N, d = 9, 4
    r = rng(17)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    dense = oracle.attention_rows(q, k, v, do, scale=0.5, causal=True, kv_len=8)
    ones = oracle.attention_rows(q, k, v, do, scale=0.5, causal=True, kv_len=8,
                                 block_mask=np.ones((3, 3)), block_size=3)
    for n in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_array_equal(dense[n], ones[n])


def test_block_diagonal_mask_factorises():
    """With only the diagonal blocks allowed, each block of rows is plain attention over
    its own block of keys."""
    N, d, bs = 8, 3, 4
    r = rng(18)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    res = oracle.attention_rows(q, k, v, do, scale=0.9, block_mask=np.eye(2), block_size=bs)
    for b in range(2):
        sl = slice(b * bs, (b + 1) * bs)
        part = oracle.attention_rows(q[sl], k[sl], v[sl], do[sl], scale=0.9)
        for n in ("o", "lse", "dq"):
            np.testing.assert_allclose(res[n][sl], part[n], atol=1e-14)
        for n in ("dk", "dv"):
            np.testing.assert_allclose(res[n][sl], part[n], atol=1e-14)


def test_block_mask_empty_rows():
    N, d = 6, 2
    r = rng(19)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    bmask = np.array([[0, 0, 0], [1, 1, 0], [0, 1, 1]])
    res = oracle.attention_rows(q, k, v, do, scale=1.0, block_mask=bmask, block_size=2)
    assert np.all(res["o"][:2] == 0) and np.all(np.isneginf(res["lse"][:2]))
    assert np.all(res["dq"][:2] == 0)
    assert np.all(np.isfinite(res["lse"][2:]))


def test_block_mask_gradients_vs_central_differences():
    N, d, bs = 6, 2, 2
    r = rng(20)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    bmask = np.array([[1, 0, 1], [1, 1, 0], [0, 1, 1]])
    kw = dict(scale=0.8, causal=False, block_mask=bmask, block_size=bs)
    res = oracle.attention_rows(q, k, v, do, **kw)

    def L(qq, kk, vv):
        return float(np.sum(oracle.attention_rows(qq, kk, vv, **kw)["o"] * do))

    eps = 1e-6
    for name, idx in (("dq", 0), ("dk", 1), ("dv", 2)):
        args = [q, k, v]
        fd = np.zeros((N, d))
        for pos in np.ndindex(N, d):
            ap = [a.copy() for a in args]
            am = [a.copy() for a in args]
            ap[idx][pos] += eps
            am[idx][pos] -= eps
            fd[pos] = (L(*ap) - L(*am)) / (2 * eps)
        assert np.linalg.norm(res[name] - fd) <= 1e-7 * max(np.linalg.norm(fd), 1.0), name
