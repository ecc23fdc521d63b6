"""Error bound of the prefill kernel's polynomial 2^x (ex2_poly), on the CPU.

The kernel evaluates part of its exponentials without the special-function
unit: n = round(x) via the 1.5 * 2^23 trick, f = x - n, a degree-3 polynomial
for 2^f, and n added to the exponent field. This test reads the coefficients
from the kernel source, repeats those float32 steps with numpy and checks the
result against 2^x in float64: relative error below 1e-4 (the fit's bound is
7.5e-5) on [-125, 8], exact zero below -125 and for -inf.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "exact_tiled_attention_38_b200", "csrc", "prefill_sm100.cuh")


def coefficients():
    text = open(SRC).read()
    c = {}
    for i in range(4):
        m = re.search(r"kExp2C%d\s*=\s*([0-9.eE+-]+)f" % i, text)
        assert m, i
        c[i] = np.float32(float(m.group(1)))
    return c


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def fma32(a, b, c):
    # a*b is exact in float64 for float32 inputs; one rounding to float32 after the add
    return f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def ex2_poly(x):
    x = f32(x)
    c = coefficients()
    magic = np.float32(12582912.0)
    with np.errstate(invalid="ignore", over="ignore"):
        t = f32(x + magic)
        n = f32(t - magic)
        f = f32(x - n)
        q = fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
        q = fma32(q, f, np.full_like(f, c[1]))
        q = fma32(q, f, np.full_like(f, c[0]))
        bits = (q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23))
        bits = ((bits + 2 ** 31) % 2 ** 32 - 2 ** 31).astype(np.int32)
        out = bits.view(np.float32)
    return np.where(x < -125.0, np.float32(0.0), out)


def test_relative_error_on_the_used_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9, 0.5),
                        [-0.5, 0.5, -1.5, 1.5, 0.0, -1e-7, 7.9999]])
    got = ex2_poly(x).astype(np.float64)
    exact = np.exp2(f32(x).astype(np.float64))
    rel = np.abs(got - exact) / exact
    assert rel.max() < 1e-4, rel.max()


def test_underflow_and_minus_infinity_give_zero():
    x = np.array([-np.inf, -1e30, -200.0, -125.5, -126.0])
    assert (ex2_poly(x) == 0).all()


def test_monotone_across_integer_boundaries():
    # continuity where n = round(x) changes (f jumps from +1/2 to -1/2)
    for k in range(-20, 8):
        lo = ex2_poly(np.array([k + 0.5 - 1e-4]))[0]
        hi = ex2_poly(np.array([k + 0.5 + 1e-4]))[0]
        assert abs(hi / lo - 2 ** 2e-4) < 2e-4
