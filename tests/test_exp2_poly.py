"""Error bound of the FMA-pipe 2^x the prefill kernel uses for one pair of exponentials in eight.

The kernel's exp2_poly (csrc/sm100.cuh) reduces x = n + f, n = round(x), evaluates
a fitted cubic for 2^f and adds n into the exponent field.  This test replays
those float32 steps with numpy over a dense grid and checks the relative error
against the exact 2^x: it must stay far below bf16's half-ulp (2^-9), since P
is rounded to bf16 right after.
"""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "heterogeneous_sliding_window_b200", "csrc", "sm100.cuh")


def _coefficients():
    text = open(HDR).read()
    body = text[text.index("float exp2_poly(float x)"):]
    body = body[:body.index("return")]
    nums = [float(x) for x in re.findall(r"fmaf\(f, (?:p|[-0-9.e+]+f), ([-0-9.e+]+)f\)", body)]
    c3 = float(re.search(r"fmaf\(f, ([-0-9.e+]+)f,", body).group(1))
    c2, c1, c0 = nums
    return np.float32(c3), np.float32(c2), np.float32(c1), np.float32(c0)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_replay(x):
    c3, c2, c1, c0 = _coefficients()
    x = np.minimum(np.maximum(x.astype(np.float32), np.float32(-125.0)), np.float32(64.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    ones = np.ones_like(f)
    p = _fma32(f, c3 * ones, c2 * ones)
    p = _fma32(f, p, c1 * ones)
    p = _fma32(f, p, c0 * ones)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_poly_coefficients_parse():
    c3, c2, c1, c0 = _coefficients()
    assert c0 == 1.0 and 0.69 < c1 < 0.70 and 0.2 < c2 < 0.3 and 0.04 < c3 < 0.07


def test_exp2_poly_relative_error():
    x = np.linspace(-124.9, 10.0, 2_000_003).astype(np.float32)
    got = exp2_poly_replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 2e-4, rel.max()
    assert rel.max() < 2.0 ** -9 / 8


def test_exp2_poly_integers_and_clamp():
    for n in range(-120, 9):
        v = exp2_poly_replay(np.array([n], dtype=np.float32))[0]
        assert abs(v / 2.0 ** n - 1.0) < 2e-4
    tiny = exp2_poly_replay(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 3e-38)
    huge = exp2_poly_replay(np.array([np.inf, 1e30, 500.0, 64.0], dtype=np.float32))
    assert np.all(np.abs(huge / 2.0 ** 64 - 1.0) < 2e-4)      # clamped, never wrapped
