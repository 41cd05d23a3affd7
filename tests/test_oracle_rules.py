"""Pins for the oracle's span rule (CPU only).

The rule itself is the "Mixture of Attention" project page, "Finding two"
(S = alpha + beta * N), rounded to the block per "Method design / Elastic
search space" and clamped to N as the heads A/B/C panel shows.
"""

import math
import os
import random
from fractions import Fraction

import pytest

from oracle import rules

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rules_project_page_heads.txt")


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, a, b, n, span, frac, note = line.split()
            rows.append((head, float(a), float(b), int(n), int(span), float(frac), note))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: r[0] + "-" + r[6])
def test_project_page_worked_heads(row):
    """The printed spans and fractions agree to the page's two significant figures."""
    head, a, b, N, printed_span, printed_frac, note = row
    S = rules.span_rule(a, b, N, 64)
    # printed to two significant figures ("1.6k", "5.6k", "0.9 * N") -> 5% relative
    assert abs(S - printed_span) <= 0.05 * printed_span + 32
    assert abs(S / N - printed_frac) <= 0.02
    if note == "clamped-to-N":
        assert S == N


def test_caption_head_b_fixed_head_c_grows():
    """Caption of the A/B/C figure: from 4k to 16k B keeps its window, C widens."""
    b4 = rules.span_rule(5600, 0.0, 4096, 64)
    b16 = rules.span_rule(5600, 0.0, 16384, 64)
    c4 = rules.span_rule(0, 0.9, 4096, 64)
    c16 = rules.span_rule(0, 0.9, 16384, 64)
    assert b4 == 4096 and b16 == rules.span_rule(5600, 0.0, 1 << 30, 64)
    assert c16 > 3.9 * c4
    # A fixed-window head does not change once N exceeds its span.
    assert rules.span_rule(1600, 0.0, 4096, 64) == rules.span_rule(1600, 0.0, 16384, 64)


def _nearest_multiple_ties_up(x, block):
    """Brute force: the multiple of block closest to x (exact rationals), ties up."""
    xf = Fraction(x)
    k0 = int(math.floor(xf / block)) - 1
    best = None
    for k in range(max(k0, 0), k0 + 4):
        cand = block * k
        dist = abs(xf - cand)
        if best is None or dist < best[0] or (dist == best[0] and cand > best[1]):
            best = (dist, cand)
    return best[1]


def test_rule_matches_brute_force_nearest_multiple():
    """Random dyadic alpha/beta: the rule equals the exact nearest multiple, clamped."""
    rnd = random.Random(1234)
    betas = [0.0, 0.125, 0.25, 0.5, 0.9, 1.0, 0.375]
    for _ in range(20000):
        block = rnd.choice([1, 16, 32, 64, 128])
        N = rnd.randint(1, 70000)
        a = rnd.randint(0, 4 * 4096) / 8.0
        b = rnd.choice(betas)
        x = a + b * N  # same two roundings the reading prescribes
        frac = Fraction(x) / block
        fpart = frac - math.floor(frac)
        if fpart != Fraction(1, 2) and abs(float(fpart) - 0.5) < 1e-9:
            continue  # binary64 evaluation of x/block + 0.5 may tie-break differently
        expect = _nearest_multiple_ties_up(x, block)
        expect = min(N, max(block, expect))
        assert rules.span_rule(a, b, N, block) == expect, (a, b, N, block)


def test_exact_tie_rounds_up():
    """5600 / 64 = 87.5 exactly: the reading rounds ties up to 88 * 64."""
    assert rules.span_rule(5600, 0.0, 16384, 64) == 5632
    assert rules.span_rule(96, 0.0, 1000, 64) == 128
    assert rules.span_rule(32, 0.0, 1000, 64) == 64  # also the lower clamp


def test_clamps():
    assert rules.span_rule(0, 0.0, 4096, 64) == 64          # lower clamp to block
    assert rules.span_rule(10, 0.0, 20, 64) == 20           # N < block -> N
    assert rules.span_rule(1e9, 1.0, 4096, 64) == 4096      # upper clamp to N
    assert rules.span_rule(0, 1.0, 300, 1) == 300


@pytest.mark.parametrize("a,b,N,blk", [
    (float("nan"), 0.0, 10, 1), (0.0, float("inf"), 10, 1), (-1.0, 0.0, 10, 1),
    (0.0, -0.5, 10, 1), (1.0, 0.0, 0, 1), (1.0, 0.0, 10, 0)])
def test_invalid_arguments(a, b, N, blk):
    with pytest.raises(ValueError):
        rules.span_rule(a, b, N, blk)


def test_monotone_in_N_and_scale():
    """Spans never shrink as N grows (alpha, beta >= 0)."""
    rnd = random.Random(7)
    for _ in range(500):
        a = rnd.choice([0, 512, 1024, 2048]) * rnd.random()
        b = rnd.choice([0, 0.125, 0.25, 0.5, 1.0])
        prev = 0
        for N in range(64, 20000, 997):
            S = rules.span_rule(a, b, N, 64)
            assert S >= min(prev, N)
            prev = S
