"""Pins of the oracle's dropout: the counter-based random numbers and their use.

Dropout sits between the softmax and the product with V in the attention op chain
(promptingindex page, "Why attention is memory-bound, not compute-bound").  Its random
numbers come from Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
As Easy as 1, 2, 3", SC 2011), a counter-based generator, so the backward pass can
regenerate the mask instead of storing it -- the same recomputation principle that the
method applies to P (anthology note "NOTE-005: FlashAttention", "Method").

What fixes the expected values here, from outside the oracle:
* the known-answer vectors published with the generator's reference library (Random123)
  and cuRAND's host-side Philox4x32-10 generator (a library routine);
* the binomial and uniform laws that an unbiased keep mask obeys;
* the definition of dropout, evaluated by brute force in numpy with the mask taken as an
  input, central finite differences through a fixed mask, and the expectation over seeds
  (E[K r] = 1 makes the mean dropped output the undropped one);
* closed forms: no dropout at p = 0, causal row 0.
"""
import ctypes
import math

import numpy as np
import pytest

import oracle


# ----------------------------------------------------------------------- Philox4x32-10

# Known-answer vectors of Philox4x32-10 from the generator's reference distribution:
# (counter, key) -> output, all words in hexadecimal.
KAT = [
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("ctr,key,out", KAT)
def test_philox_known_answers(ctr, key, out):
    assert oracle.philox4x32_10(ctr, key) == list(out)


def _curand():
    for name in ("libcurand.so", "libcurand.so.10"):
        try:
            return ctypes.CDLL(name)
        except OSError:
            continue
    return None


def test_philox_matches_curand_host_generator():
    """cuRAND's host generator CURAND_RNG_PSEUDO_PHILOX4_32_10 (enum 161) with seed 0
    emits, four words at a time, Philox4x32-10 of key (0, 0) and counters (0, 0, n, 0)."""
    lib = _curand()
    if lib is None:
        pytest.skip("libcurand is not loadable here")
    gen = ctypes.c_void_p()
    if lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) != 0:
        pytest.skip("cuRAND host generator unavailable")
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(0)) == 0
        words = np.zeros(32, dtype=np.uint32)
        assert lib.curandGenerate(gen, words.ctypes.data_as(ctypes.c_void_p),
                                  ctypes.c_size_t(words.size)) == 0
    finally:
        lib.curandDestroyGenerator(gen)
    for n in range(8):
        assert oracle.philox4x32_10((0, 0, n, 0), (0, 0)) == [int(x) for x in words[4 * n:4 * n + 4]]


def test_philox_bijective_on_a_sample():
    """A Philox round function is a bijection of the counter for a fixed key: 4096
    distinct counters give 4096 distinct outputs."""
    outs = {tuple(oracle.philox4x32_10((c & 7, c >> 3, 5, 0), (1, 2))) for c in range(4096)}
    assert len(outs) == 4096


# ----------------------------------------------------------------------- the mask


def test_threshold_rule():
    assert oracle.dropout_threshold(0.0) == 0
    assert oracle.dropout_threshold(0.1) == 26       # 25.6 -> 26
    assert oracle.dropout_threshold(0.5) == 128
    assert oracle.dropout_threshold(0.5 / 256) == 0  # tie -> even
    assert oracle.dropout_threshold(1.5 / 256) == 2  # tie -> even
    assert oracle.dropout_threshold(255.4 / 256) == 255
    for bad in (-0.01, 255.6 / 256, 1.0, 2.0):
        with pytest.raises(ValueError):
            oracle.dropout_threshold(bad)


def test_mask_layout_is_the_stated_one():
    """Element (i, j) of head bh is decided by byte j mod 16 of the Philox output for
    counter (j // 16, i, bh, offset), key (seed low word, seed high word)."""
    seed, off, bh = 0x0123456789ABCDEF, 7, 3
    keep = oracle.dropout_keep(0.3, seed, off, bh, 9, 70)
    t = oracle.dropout_threshold(0.3)
    for i in range(9):
        for j in range(70):
            w = oracle.philox4x32_10((j // 16, i, bh, off), (seed & 0xFFFFFFFF, seed >> 32))
            byte = (w[(j % 16) // 4] >> (8 * (j % 4))) & 0xFF
            assert byte == oracle.dropout_byte(seed, off, bh, i, j)
            assert keep[i, j] == (byte >= t)


def test_bytes_uniform_and_keep_rate_binomial():
    """Over 2^17 elements the bytes pass a chi-square test for uniformity, and for several
    thresholds the kept fraction lies within 6 sigma of (256 - t) / 256."""
    n_q, n_k = 128, 1024
    counts = np.zeros(256)
    for t in (26, 128, 230):
        p = t / 256
        keep = oracle.dropout_keep(p, 1234, 0, 5, n_q, n_k)
        q = (256 - t) / 256
        sd = math.sqrt(q * (1 - q) / keep.size)
        assert abs(keep.mean() - q) < 6 * sd, (t, keep.mean(), q)
        # adjacent keys of one 16-key group are independent: P(both kept) = q^2
        both = (keep[:, 0::2] & keep[:, 1::2]).mean()
        sd2 = math.sqrt(q * q * (1 - q * q) / (keep.size // 2))
        assert abs(both - q * q) < 6 * sd2, (t, both, q * q)
    # byte histogram from the thresholds' cumulative counts: P(byte >= t) for every t
    ge = np.array([oracle.dropout_keep(t / 256, 99, 1, 0, 64, 512).sum() for t in range(256)]
                  + [0], dtype=np.float64)
    counts = ge[:-1] - ge[1:]
    n = 64 * 512
    chi2 = ((counts - n / 256) ** 2 / (n / 256)).sum()
    assert chi2 < 255 + 6 * math.sqrt(2 * 255), chi2


def test_streams_differ():
    """Different seeds, offsets, heads or rows give (almost surely) different masks."""
    base = oracle.dropout_keep(0.5, 1, 0, 0, 4, 256)
    for args in ((2, 0, 0), (1, 1, 0), (1, 0, 1), (1 << 32 | 1, 0, 0)):
        other = oracle.dropout_keep(0.5, args[0], args[1], args[2], 4, 256)
        assert (other != base).mean() > 0.3, args
    assert (base[0] != base[1]).mean() > 0.3


# ----------------------------------------------------------------------- dropout in attention


def rng(seed):
    return np.random.default_rng(seed)


def brute_dropout(q, k, v, scale, causal, L, keep, r):
    N = q.shape[0]
    S = scale * (q @ k.T)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    allowed = (j < L) & ((not causal) | (j <= i))
    E = np.where(allowed, np.exp(np.where(allowed, S, 0.0)), 0.0)
    Z = E.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        P = np.where(Z[:, None] > 0, E / Z[:, None], 0.0)
        lse = np.where(Z > 0, np.log(Z), -np.inf)
    return (P * keep * r) @ v, lse


@pytest.mark.parametrize("N,d,causal,L,p", [(5, 3, False, 5, 0.25), (8, 4, True, 8, 0.5),
                                            (7, 2, True, 4, 0.1), (33, 4, False, 30, 0.75)])
def test_brute_force_with_mask_as_input(N, d, causal, L, p):
    r_ = rng(N * 7 + d)
    q, k, v = (r_.standard_normal((N, d)) for _ in range(3))
    seed, off, bh = 77, 3, 2
    keep = oracle.dropout_keep(p, seed, off, bh, N, N).astype(np.float64)
    t = oracle.dropout_threshold(p)
    res = oracle.attention_rows(q, k, v, scale=0.8, causal=causal, kv_len=L, dropout_p=p,
                                seed=seed, offset=off, bh=bh)
    o_bf, lse_bf = brute_dropout(q, k, v, 0.8, causal, L, keep, 256 / (256 - t))
    np.testing.assert_allclose(res["o"], o_bf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(res["lse"], lse_bf, rtol=1e-12, atol=1e-13)


def test_zero_probability_is_no_dropout():
    r_ = rng(5)
    q, k, v, do = (r_.standard_normal((20, 4)) for _ in range(4))
    a = oracle.attention_rows(q, k, v, do, scale=0.5, causal=True, kv_len=17)
    b = oracle.attention_rows(q, k, v, do, scale=0.5, causal=True, kv_len=17, dropout_p=0.0,
                              seed=123)
    for name in a:
        assert np.array_equal(a[name], b[name]), name


def test_causal_row_zero_closed_form():
    """Row 0 under causal masking sees key 0 only: P_00 = 1, so O_0 = K_00 r v_0 and
    LSE_0 = scale q_0 . k_0 whether or not the element is dropped."""
    r_ = rng(6)
    q, k, v = (r_.standard_normal((16, 4)) for _ in range(3))
    p = 0.5
    hits = set()
    for seed in range(12):
        res = oracle.attention_rows(q, k, v, scale=0.9, causal=True, dropout_p=p, seed=seed)
        kept = oracle.dropout_keep(p, seed, 0, 0, 1, 1)[0, 0]
        hits.add(int(kept))
        np.testing.assert_allclose(res["o"][0], v[0] * 2.0 * kept, atol=1e-14)
        np.testing.assert_allclose(res["lse"][0], 0.9 * q[0] @ k[0], rtol=1e-14)
    assert hits == {0, 1}


def loss(q, k, v, do, scale, causal, L, p, seed):
    return float((oracle.attention_rows(q, k, v, scale=scale, causal=causal, kv_len=L,
                                        dropout_p=p, seed=seed, offset=1, bh=4)["o"] * do).sum())


@pytest.mark.parametrize("N,d,causal,L,p", [(6, 3, False, 6, 0.3), (7, 4, True, 5, 0.5),
                                            (8, 2, True, 8, 0.2)])
def test_gradients_finite_differences(N, d, causal, L, p):
    """Central differences of sum(O * dO) through a fixed mask (the seed fixes it)."""
    r_ = rng(100 + N)
    q, k, v, do = (r_.standard_normal((N, d)) for _ in range(4))
    scale, seed, eps = 0.6, 2024, 1e-6
    res = oracle.attention_rows(q, k, v, do, scale=scale, causal=causal, kv_len=L, dropout_p=p,
                                seed=seed, offset=1, bh=4)
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        g = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            old = x[idx]
            x[idx] = old + eps
            lp_ = loss(q, k, v, do, scale, causal, L, p, seed)
            x[idx] = old - eps
            lm = loss(q, k, v, do, scale, causal, L, p, seed)
            x[idx] = old
            g[idx] = (lp_ - lm) / (2 * eps)
        err = np.linalg.norm(res[name] - g) / max(np.linalg.norm(g), 1e-300)
        assert err < 1e-6, (name, err)


def test_expectation_over_seeds_is_undropped_output():
    """E[K r] = 1 per element, so the mean over seeds of the dropped output tends to the
    undropped output; with 2000 seeds the gap is within 6 standard errors."""
    r_ = rng(8)
    N, d, p = 6, 3, 0.5
    q, k, v = (r_.standard_normal((N, d)) for _ in range(3))
    ref = oracle.attention_rows(q, k, v, scale=1.0)["o"]
    outs = np.stack([oracle.attention_rows(q, k, v, scale=1.0, dropout_p=p, seed=s)["o"]
                     for s in range(2000)])
    se = outs.std(axis=0) / math.sqrt(outs.shape[0])
    assert np.all(np.abs(outs.mean(axis=0) - ref) < 6 * se + 1e-12)


def test_full_tensor_interface_uses_head_index():
    """attention() draws head (b, h)'s mask as bh = b * H + h."""
    r_ = rng(9)
    B, H, N, d = 2, 3, 12, 4
    q, k, v = (r_.standard_normal((B, H, N, d)) for _ in range(3))
    full = oracle.attention(q, k, v, scale=0.5, dropout_p=0.4, seed=11, offset=2)
    for b in range(B):
        for h in range(H):
            one = oracle.attention_rows(q[b, h], k[b, h], v[b, h], scale=0.5, dropout_p=0.4,
                                        seed=11, offset=2, bh=b * H + h)
            assert np.array_equal(full["o"][b, h], one["o"])
