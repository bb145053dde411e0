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


# ---------------------------------------------------------------- FP4 and Int4
# "1. 4-bit NormalFloat (NF4)" names Integer 4-bit and Float 4-bit as the
# usual alternatives and says NF4 has the lower quantization error
# ("Performance and Evaluation": "NF4 efficiency").  The readings (oracle
# header): FP4 = the 1-sign 2-exponent 1-mantissa float divided by its
# largest magnitude 6; Int4 = k/7.  Pinned here against their values written
# out as rationals (not derived from bit fields as the oracle does).
from fractions import Fraction  # noqa: E402

from oracle import fp4_codebook, int4_codebook, quantize_nf4, dequantize_nf4, bf16_round  # noqa: E402
from tests.exact import frac, rn_f32  # noqa: E402

FP4_POS = [Fraction(1, 12), Fraction(1, 6), Fraction(1, 4), Fraction(1, 3), Fraction(1, 2), Fraction(2, 3),
           Fraction(1)]  # 0.5, 1, 1.5, 2, 3, 4, 6 over 6
FP4_RAT = [-v for v in reversed(FP4_POS)] + [Fraction(0)] + FP4_POS + [Fraction(1)]
INT4_RAT = [Fraction(k, 7) for k in range(-7, 8)] + [Fraction(1)]


def _layout_invariants(q):
    assert q.dtype == np.float32 and q.shape == (16,)
    assert np.all(np.diff(q[:15]) > 0), "strictly increasing over the 15 distinct levels"
    assert q[0] == -1.0 and q[7] == 0.0 and q[14] == 1.0 and q[15] == 1.0
    assert np.sum(q < 0) == 7 and np.sum(q[:15] > 0) == 7


def test_fp4_levels_are_the_float_values_over_six():
    q = fp4_codebook()
    _layout_invariants(q)
    assert [frac(v) for v in q] == [rn_f32(v) for v in FP4_RAT]


def test_int4_levels_are_k_over_7():
    q = int4_codebook()
    _layout_invariants(q)
    assert [frac(v) for v in q] == [rn_f32(v) for v in INT4_RAT]


def test_nf4_has_the_lowest_error_on_normally_distributed_weights():
    """The pages' claim, on N(0, 0.02^2) weights: NF4's mean squared
    quantization error is below FP4's and Int4's (same blocks, same double
    quantization)."""
    rng = np.random.default_rng(2024)
    x = bf16_round(rng.standard_normal(64 * 4096).astype(np.float32) * np.float32(0.02))
    mse = {}
    for code in ("nf4", "fp4", "int4"):
        p, a, c = quantize_nf4(x, code=code)
        w = dequantize_nf4(p, a, c, x.size, code=code).astype(np.float64)
        mse[code] = float(np.mean((w - x) ** 2))
        if code != "nf4":
            nib = np.concatenate([p >> 4, p & 15])
            assert not np.any(nib == 15), "the repeated top level is never chosen"
    assert mse["nf4"] < mse["fp4"] and mse["nf4"] < mse["int4"], mse
