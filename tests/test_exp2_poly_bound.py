"""Error bound of the attention kernel's FMA-pipe exp2.

The kernel evaluates part of the softmax exponentials 2^x (x <= 0, clamped at
-126) without the MUFU: x = j + f with j = round(x) obtained by adding
1.5 * 2^23, 2^f by a cubic in f on [-1/2, 1/2] (Horner with fused
multiply-adds), and j added to the exponent field of the result. Its source
states a maximum relative error of 7.7e-5 wherever 2^x is a normal float32
(x >= -125; bf16, which stores P, keeps 3.9e-3). This test reads the cubic's coefficients from the kernel source (the packed
form computes two values with the same fused multiply-adds, so each lane's
arithmetic is what is evaluated here),
evaluates the same float32 steps on the host over a dense grid of
[-126, 0] and over every float32 f in a fine grid of [-1/2, 1/2], and checks the
stated bound against numpy's float64 exp2.
"""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "audio_generation_b200", "csrc", "attention.cu")
STATED_MAX_REL = 7.7e-5


def _coefficients():
    """The cubic's coefficients kExpC3 .. kExpC0 as the kernel source states them."""
    src = open(SRC).read()
    vals = {}
    for name in ("kExpC3", "kExpC2", "kExpC1", "kExpC0"):
        m = re.search(name + r"\s*=\s*(-?\d+\.\d+)f", src)
        assert m, name
        vals[name] = float(m.group(1))
    assert re.search(r"kRoundMagic\s*=\s*12582912\.f", src)
    return vals["kExpC3"], vals["kExpC2"], vals["kExpC1"], vals["kExpC0"]


def _fma32(a, b, c):
    # float32 operands: the float64 product is exact, one rounding to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_host(x):
    c3, c2, c1, c0 = (np.float32(c) for c in _coefficients())
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = _fma32(_fma32(_fma32(np.full_like(f, c3), f, np.full_like(f, c2)), f,
                      np.full_like(f, c1)), f, np.full_like(f, c0))
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.int32).view(np.float32)


def test_exp2_poly_relative_error_within_stated_bound():
    g = np.random.default_rng(0)
    xs = [np.linspace(-126.0, 0.0, 2_000_001, dtype=np.float64).astype(np.float32),
          g.uniform(-126.0, 0.0, 1_000_000).astype(np.float32)]
    f = np.linspace(-0.5, 0.5, 200_001, dtype=np.float64)
    for j in (0, -1, -7, -40, -125):
        xs.append((j + f).astype(np.float32))
    x = np.concatenate(xs)
    x = x[(x >= -126.0) & (x <= 0.0)]
    got = exp2_poly_host(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(got))
    normal = x >= -125.0  # results that are normal float32 values
    rel = np.abs(got[normal] - want[normal]) / want[normal]
    assert rel.max() <= STATED_MAX_REL * 1.01, rel.max()
    # a cubic, not exact: the bound is attained to within a few percent
    assert rel.max() > 0.9 * STATED_MAX_REL
    # below 2^-125 the exponent step leaves the normal range; the error there is
    # absolute and negligible next to a softmax row sum (>= 1)
    assert np.abs(got[~normal] - want[~normal]).max() <= 2.0 ** -135


def test_exp2_poly_special_points():
    x = np.array([0.0, -1.0, -0.5, -126.0, -200.0, -1e30], np.float32)
    got = exp2_poly_host(x).astype(np.float64)
    np.testing.assert_allclose(got[:3], np.exp2(x[:3].astype(np.float64)), rtol=1e-4)
    # clamped: inputs below -126 give 2^-126 times the cubic at 0, tiny next to a row sum >= 1
    assert np.all(got[3:] > 0) and np.all(got[3:] < 2.0 ** -125)
