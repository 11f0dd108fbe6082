"""The polynomial 2^x that the d = 64 forward kernel evaluates on the FMA pipe for part of
each softmax row (exp2_poly2 in exact_io_aware_60_b200/csrc/sm100.cuh), checked on the CPU
from the constants in that header: the range reduction x = n + f, n = round(x), f in
[-1/2, 1/2], and the degree-3 polynomial for 2^f, evaluated in fp32 as the kernel does.
The relative error must stay below 8e-5 (13.6 bits; the 16-bit P it feeds keeps 8 or 11)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_io_aware_60_b200", "csrc", "sm100.cuh")


def constants():
    src = open(HDR, encoding="utf-8").read()
    c = {}
    for name in ("kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3", "kRoundMagic"):
        m = re.search(rf"constexpr float {name} = ([0-9.eE+-]+)f;", src)
        assert m, name
        c[name] = np.float32(float(m.group(1)))
    return c


def exp2_poly(x):
    """The kernel's steps in fp32: clamp, round by the magic constant, polynomial, add n
    to the exponent field."""
    c = constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + c["kRoundMagic"]).astype(np.float32)
    n = (t - c["kRoundMagic"]).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c["kExp2C3"] * f + c["kExp2C2"]).astype(np.float32)
    p = (p * f + c["kExp2C1"]).astype(np.float32)
    p = (p * f + c["kExp2C0"]).astype(np.float32)
    bits = (t.view(np.uint32).astype(np.uint64) * (1 << 23) + p.view(np.uint32)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-125.0, 0.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 8e-5, rel.max()
    # the bound is that of the polynomial on [-1/2, 1/2], not of a lucky grid
    assert rel.max() > 5e-5


def test_exact_at_integers_up_to_the_polynomial_error_and_clamped_below():
    x = np.arange(-125, 1, dtype=np.float32)
    got = exp2_poly(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) < 8e-5)
    # below the clamp the result is about 2^-125: a normal number, zero for a 16-bit P
    # next to any visible key (whose P is at least 2^-8 of the row's largest)
    low = exp2_poly(np.array([-126.0, -1e4, -np.inf], dtype=np.float32)).astype(np.float64)
    assert np.all(np.abs(low / 2.0 ** -125 - 1) < 8e-5)
