"""The comparison helpers of the GPU parity tests, checked on CPU."""
import numpy as np
import torch

from parity import O_ATOL, O_EPS, half_ulp, head_rel_l2_max, o_graded_error, rel_l2, rounding_floor


def test_half_ulp_bounds_actual_rounding():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 1.0, 7.0, 300.0)])
    for dt in (torch.bfloat16, torch.float16):
        # torch rounds fp64 -> fp32 -> 16 bits; the double rounding can exceed half an
        # ulp by at most 2^-13 of an ulp
        r = torch.from_numpy(x).to(dt).double().numpy()
        err = np.abs(r - x)
        h = half_ulp(x, dt)
        assert np.all(err <= h * (1 + 2.0 ** -12))
        assert np.max(err / h) > 0.99           # the bound is attained
        assert rounding_floor(x, dt) == np.max(err)


def test_o_graded_error_is_plain_max_abs_below_4():
    # Where half an ulp plus O_EPS fits under O_ATOL (|O| < 4 in bf16, < 8 in fp16) the
    # grade is the plain absolute error: 0.0105 fails at every such magnitude, even where
    # half an ulp alone is 0.0078 (bf16 in [2, 4)).
    for dt, top in ((torch.bfloat16, 4.0), (torch.float16, 8.0)):
        ref = np.array([0.01, 0.5, 1.5, 2.5, 3.9, top * 0.99])
        for delta in (0.0042, -0.0099):
            assert abs(o_graded_error(ref + delta, ref, dt) - abs(delta)) < 1e-15
        assert o_graded_error(ref + 0.0105, ref, dt) > O_ATOL


def test_o_graded_error_large_values():
    # |O| in [4, 8) in bf16: spacing 2^-5, so exact rounding alone errs by up to 2^-6
    ref = np.array([4.0 + 2.0 ** -6, 5.0 + 2.0 ** -6 - 1e-9, 7.5])
    out = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert np.max(np.abs(out - ref)) > O_ATOL              # the plain bound cannot hold
    assert o_graded_error(out, ref, torch.bfloat16) <= O_ATOL   # the graded one does
    # the allowance there is exactly half an ulp + O_EPS, and no more
    ulp_half = 2.0 ** -6
    assert o_graded_error(ref + ulp_half + O_EPS - 1e-6, ref, torch.bfloat16) <= O_ATOL
    assert o_graded_error(ref + ulp_half + O_EPS + 1e-4, ref, torch.bfloat16) > O_ATOL


def test_rel_l2():
    a = np.array([3.0, 4.0])
    assert rel_l2(a, a) == 0.0
    assert abs(rel_l2(a * 1.01, a) - 0.01) < 1e-12


def test_head_rel_l2_max_finds_a_local_error():
    rng = np.random.default_rng(1)
    r = rng.standard_normal((4, 6, 256, 64))
    g = r * (1 + 1e-3 * rng.standard_normal(r.shape))
    assert head_rel_l2_max(g, r) < 2e-3
    # a 32-row error of 10% in one head: invisible in the norm over all 24 heads at 2e-2,
    # visible per head
    bad = g.copy()
    bad[2, 3, 100:132] *= 1.1
    assert rel_l2(bad, r) < 2e-2
    assert head_rel_l2_max(bad, r) > 2e-2


def test_head_rel_l2_max_zero_reference_head():
    # a head whose exact gradient is zero is measured against the RMS head norm
    rng = np.random.default_rng(2)
    r = rng.standard_normal((3, 128, 64))
    r[1] = 0.0
    g = r.copy()
    g[1] = 1e-4
    rms = np.sqrt(np.sum(r ** 2) / 3)
    assert abs(head_rel_l2_max(g, r) - np.sqrt(128 * 64) * 1e-4 / rms) < 1e-12


def test_o_graded_error_with_an_output_scale():
    # s = 10 (dropout p = 0.9): the grade is that of O / s, with the output's own half ulp
    ref = np.array([0.5, 2.5, 30.0])
    assert o_graded_error(ref + 0.05, ref, torch.bfloat16, 10.0) == 0.005 or \
        abs(o_graded_error(ref + 0.05, ref, torch.bfloat16, 10.0) - 0.005) < 1e-12
    assert o_graded_error(ref + 0.11, ref, torch.bfloat16, 10.0) > O_ATOL
    # at |O| = 30 (bf16 spacing 0.125) exact rounding passes
    out = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert o_graded_error(out, ref, torch.bfloat16, 10.0) <= O_ATOL
