"""Pins for the oracle's NF4 codebook.

The pages ("1. 4-bit NormalFloat (NF4)" in "QLoRA: Fine-Tuning 65-Billion
Parameter Models ..."; "AI Glossary: QLoRA", second paragraph) say only that
NF4 suits normally distributed values and gives every bucket an equal share;
the exact zero and +-1 endpoints are part of the chosen reading.  No table is
printed, so the numbers themselves are pinned to the reading: invariants,
a second normal-quantile route (bisection on erfc instead of the standard
library's rational approximation) and the equal-probability spacing checked
with erf.
"""

import math

import numpy as np

from oracle import nf4_codebook

DELTA = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)


def phi(x):
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def quantile_bisect(p):
    lo, hi = -40.0, 40.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_invariants():
    q = nf4_codebook()
    assert q.dtype == np.float32 and q.shape == (16,)
    assert np.all(np.diff(q) > 0), "strictly increasing"
    assert q[0] == -1.0 and q[15] == 1.0 and q[7] == 0.0
    assert np.sum(q < 0) == 7 and np.sum(q > 0) == 8
    assert np.all(np.abs(q) <= 1.0)


def test_second_quantile_route_matches_in_float32():
    z = quantile_bisect(DELTA)
    pos = [quantile_bisect(0.5 + j * (DELTA - 0.5) / 8.0) / z for j in range(1, 9)]
    neg = [-quantile_bisect(0.5 + j * (DELTA - 0.5) / 7.0) / z for j in range(1, 8)]
    ref = np.array(sorted(neg + [0.0] + pos), dtype=np.float64).astype(np.float32)
    np.testing.assert_array_equal(nf4_codebook(), ref)


def test_equal_probability_spacing_per_side():
    q = nf4_codebook().astype(np.float64)
    z = quantile_bisect(DELTA)
    pos_p = [phi(v * z) for v in q[7:]]          # 0, q8 .. q15
    neg_p = [phi(-v * z) for v in q[7::-1]]      # 0, -q6 .. -q0
    np.testing.assert_allclose(np.diff(pos_p), (DELTA - 0.5) / 8.0, rtol=0, atol=2e-7)
    np.testing.assert_allclose(np.diff(neg_p), (DELTA - 0.5) / 7.0, rtol=0, atol=2e-7)


def test_max_half_gap_is_between_the_two_lowest_levels():
    q = nf4_codebook().astype(np.float64)
    gaps = np.diff(q)
    assert int(np.argmax(gaps)) == 0
    assert abs(gaps.max() / 2 - 0.1519) < 1e-4
