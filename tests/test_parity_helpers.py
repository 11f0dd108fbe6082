"""The comparison helpers of the GPU parity tests, checked on CPU."""
import numpy as np
import torch

from parity import half_ulp, o_error_beyond_rounding, rel_l2, rounding_floor


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


def test_o_error_beyond_rounding():
    ref = np.array([0.5, 5.0])
    # an exactly rounded output has no error beyond rounding
    out = torch.from_numpy(ref + 0.013).to(torch.bfloat16).double().numpy()
    e = o_error_beyond_rounding(out, ref + 0.013, torch.bfloat16)
    assert e <= 1e-12
    # a computation error of 0.02 on top of rounding is visible
    assert o_error_beyond_rounding(ref + 0.02, ref, torch.bfloat16) > 0.004


def test_rel_l2():
    a = np.array([3.0, 4.0])
    assert rel_l2(a, a) == 0.0
    assert abs(rel_l2(a * 1.01, a) - 0.01) < 1e-12
