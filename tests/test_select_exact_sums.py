"""The selection filter's parallel walk rests on one fact: fp32 values that lie
within 19 binades of one another, at most 256 of them, have fp64 partial sums
that are all exact, so the sums do not depend on the order of the additions.
The filter's candidates are exactly such sets (theta is a power of two at
least m * 2^-18 below the row maximum m), and the definition of find_blocks
adds them one after another in fp64. These tests check the fact on the host:
the one-by-one fp64 prefix sums of ranked candidates equal, bit for bit, the
prefix sums of a Hillis-Steele scan (the order a warp scan adds in) and the
exact rational sums. A control with a wider span shows that the property is
not automatic.
"""
from fractions import Fraction

import numpy as np
import pytest


def _candidates(rng, n, shift):
    """fp32 values of a synthetic probability row and its filter candidates
    for theta = 2^(e_max - shift) (e_max: the row maximum's binade)."""
    row = rng.pareto(1.2, size=n).astype(np.float32) * rng.random(n).astype(np.float32)
    row = (row / row.sum()).astype(np.float32)
    m = float(row.max())
    theta = np.float32(2.0 ** (np.floor(np.log2(m)) - shift))
    cand = np.sort(row[row >= theta])[::-1]
    return cand


def _sequential(c):
    out, acc = [], 0.0
    for v in c:
        acc = acc + float(v)   # fp64, one after another
        out.append(acc)
    return np.array(out)


def _hillis_steele(c):
    x = c.astype(np.float64).copy()
    step = 1
    while step < len(x):
        y = x.copy()
        y[step:] = x[step:] + x[:-step]
        x = y
        step *= 2
    return x


@pytest.mark.parametrize("seed", range(40))
@pytest.mark.parametrize("shift", [6, 12, 18])
def test_prefix_sums_are_exact_within_19_binades(seed, shift):
    rng = np.random.default_rng(seed)
    c = _candidates(rng, int(rng.integers(64, 4096)), shift)[:256]
    if len(c) == 0:
        return
    seq = _sequential(c)
    assert np.array_equal(seq, _hillis_steele(c))
    exact = np.cumsum([Fraction(float(v)) for v in c])
    assert all(Fraction(float(s)) == e for s, e in zip(seq, exact))


def test_a_wider_span_can_round():
    """Control: over a span of 60 binades an fp64 sum of fp32 values rounds
    (the smaller term is lost), so the bound on the span is what makes the
    sums exact."""
    big, tiny = np.float32(1.0), np.float32(2.0 ** -60)
    s = float(big) + float(tiny)
    assert s == 1.0
    assert Fraction(float(big)) + Fraction(float(tiny)) != Fraction(s)
