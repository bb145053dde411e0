"""Pins for the oracle's NF4 quantize / double-quant / dequantize.

Each pin recomputes a result by a route that shares nothing with the
oracle's numpy code: exact rational arithmetic (fractions.Fraction) with
rounding to float32/bfloat16 done by integer arithmetic (tests/exact.py),
nearest-level search by comparing exact distances, and a nibble/byte layout
rebuilt element by element.  Closed forms and special cases come from the
pages: "AI Glossary: QLoRA", second paragraph, and "2. Double Quantization"
in "QLoRA: Fine-Tuning 65-Billion Parameter Models ..." (about 0.37 bits per
parameter saved, about 3 GB at 65B parameters).
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4_codebook, quantize_nf4, dequantize_nf4, dequantize_scales, dequantize_at, bf16_round
from oracle.nf4_ref import bits_per_parameter, max_half_gap
from tests.exact import frac, rn_f32, rn_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
Q = [frac(v) for v in nf4_codebook()]
L2 = [rn_f32(Fraction(k, 255)) for k in range(256)]
# The FP4 and Int4 readings written out as rationals (see
# tests/test_oracle_codebook.py), rounded to float32 exactly.
_FP4_POS = [Fraction(1, 12), Fraction(1, 6), Fraction(1, 4), Fraction(1, 3), Fraction(1, 2), Fraction(2, 3),
            Fraction(1)]
LEVELS = {
    "nf4": Q,
    "fp4": [rn_f32(v) for v in [-v for v in reversed(_FP4_POS)] + [Fraction(0)] + _FP4_POS + [Fraction(1)]],
    "int4": [rn_f32(Fraction(k, 7)) for k in list(range(-7, 8)) + [7]],
}


def nearest(value, levels):
    best, best_d = 0, None
    for i, lv in enumerate(levels):
        d = abs(value - lv)
        if best_d is None or d < best_d:
            best, best_d = i, d
    return best


def brute_quantize(x, block=64, group=256, levels=None):
    """Element-by-element restatement of the codec (exact rationals)."""
    levels = Q if levels is None else levels
    xs = [frac(v) for v in x]
    n = len(xs)
    nb = -(-n // block)
    c = [max(abs(v) for v in xs[b * block:(b + 1) * block]) for b in range(nb)]
    codes = []
    for i, v in enumerate(xs):
        cb = c[i // block]
        codes.append(7 if cb == 0 else nearest(rn_f32(v / cb), levels))
    if n % 2:
        codes.append(7)
    packed = [codes[2 * j] * 16 + codes[2 * j + 1] for j in range(len(codes) // 2)]
    nb2 = -(-nb // group)
    c1 = [max(c[g * group:(g + 1) * group]) for g in range(nb2)]
    code2 = []
    for b in range(nb):
        m = c1[b // group]
        code2.append(0 if m == 0 else nearest(rn_f32(c[b] / m), L2))
    return packed, code2, c1


def brute_dequantize(packed, code2, c1, n, block=64, group=256, levels=None):
    levels = Q if levels is None else levels
    nib = []
    for byte in packed:
        nib += [byte >> 4, byte & 15]
    out = []
    for i in range(n):
        b = i // block
        a = rn_f32(L2[code2[b]] * c1[b // group])
        out.append(rn_bf16(rn_f32(levels[nib[i]] * a)))
    return out


def bf16_values(rng, n, std):
    return bf16_round(rng.standard_normal(n).astype(np.float32) * np.float32(std))


# NF4 on every size; the other codebooks on a subset of them.
BRUTE_CASES = ([("nf4", n) for n in (1, 2, 63, 64, 65, 127, 130, 64 * 256 + 5)]
               + [(c, n) for c in ("fp4", "int4") for n in (1, 65, 64 * 256 + 5)])


@pytest.mark.parametrize("code,n", BRUTE_CASES)
def test_quantize_matches_brute_force(n, code):
    rng = np.random.default_rng(100 + n)
    x = bf16_values(rng, n, 0.02)
    if n > 70:
        x[64:128] = 0.0  # an all-zero block
    packed, code2, c1 = quantize_nf4(x, code=code)
    bp, bc2, bc1 = brute_quantize(list(x), levels=LEVELS[code])
    assert packed.tolist() == bp
    assert code2.tolist() == bc2
    assert [frac(v) for v in c1] == bc1


@pytest.mark.parametrize("code", ["nf4", "fp4", "int4"])
def test_dequantize_matches_brute_force(code):
    rng = np.random.default_rng(7)
    n = 64 * 256 + 37
    x = bf16_values(rng, n, 0.05)
    packed, code2, c1 = quantize_nf4(x, code=code)
    got = dequantize_nf4(packed, code2, c1, n, code=code)
    ref = brute_dequantize(packed.tolist(), code2.tolist(), [frac(v) for v in c1], n, levels=LEVELS[code])
    assert [frac(v) for v in got] == ref


@pytest.mark.parametrize("code", ["nf4", "fp4", "int4"])
def test_every_bf16_pattern_against_exact_threshold(code):
    """All finite bf16 values x with |x| <= c, for several block maxima c
    (including ones whose quotient x/c is not a float32, so the rounding of
    the scaled value matters), against exact midpoint counting."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    allv = bits.view(np.float32)
    allv = allv[np.isfinite(allv)]
    lv = LEVELS[code]
    mids = [(lv[i] + lv[i + 1]) / 2 for i in range(15)]
    for c in ((1.0, 0.75, 0.0234375, 3.0) if code == "nf4" else (0.75, 3.0)):
        xs = allv[np.abs(allv) <= c]
        # Blocks of 64: [c, x, x, ..., x] so the block absmax is exactly c.
        blocks = np.repeat(xs[:, None], 64, axis=1)
        blocks[:, 0] = c
        packed, _, _ = quantize_nf4(blocks.reshape(-1), code=code)
        codes = (packed.reshape(-1, 32)[:, 0] & 15)  # element 1 of each block
        cf = Fraction(c)
        for x, got in zip(xs.tolist(), codes.tolist()):
            nq = rn_f32(Fraction(x) / cf)
            ref = sum(1 for m in mids if nq > m)  # ties -> lower index
            assert got == ref, (c, x, got, ref)


def test_special_cases():
    x = np.zeros(128, np.float32)
    x[:64] = bf16_round(np.linspace(-0.5, 0.25, 64).astype(np.float32))
    packed, code2, c1 = quantize_nf4(x)
    codes = np.stack([packed >> 4, packed & 15], axis=1).reshape(-1)
    assert codes[0] == 0          # x = -c_b -> lowest level
    assert np.all(codes[64:] == 7)  # all-zero block -> zero level
    assert code2[0] == 255 and code2[1] == 0  # group max -> 255; zero block -> 0
    x2 = x.copy()
    x2[5] = 0.5
    packed2, _, _ = quantize_nf4(x2)
    assert (packed2[2] & 15) == 15  # element 5 (low nibble of byte 2): x = +c_b -> highest level
    w = dequantize_nf4(packed, code2, c1, 128)
    assert w[0] == -0.5           # a' = c1 exactly when code2 == 255
    assert np.all(w[64:] == 0.0)


def test_group_max_constant_is_exact():
    rng = np.random.default_rng(3)
    x = bf16_values(rng, 64 * 512, 0.02)
    packed, code2, c1 = quantize_nf4(x)
    a = dequantize_scales(code2, c1)
    c = np.abs(x).reshape(-1, 64).max(axis=1)
    for g in range(2):
        seg = slice(g * 256, (g + 1) * 256)
        j = int(np.argmax(c[seg]))
        assert code2[seg][j] == 255 and a[seg][j] == c1[g] == c[seg][j]


def test_level2_nearest_code_brute_force_all_levels():
    rng = np.random.default_rng(11)
    c = bf16_round(np.abs(rng.standard_normal(256 * 3).astype(np.float32)) * np.float32(0.03))
    # Build blocks whose absmax is exactly c_b: one element = c_b, rest small.
    x = np.zeros((c.size, 64), np.float32)
    x[:, 0] = c
    _, code2, c1 = quantize_nf4(x.reshape(-1))
    for b in range(c.size):
        m = Fraction(float(c1[b // 256]))
        ref = nearest(rn_f32(Fraction(float(c[b])) / m), L2)
        assert code2[b] == ref


def test_dequant_error_bound():
    rng = np.random.default_rng(5)
    n = 64 * 1024
    x = bf16_values(rng, n, 0.02)
    packed, code2, c1 = quantize_nf4(x)
    w = dequantize_nf4(packed, code2, c1, n).astype(np.float64)
    a = np.repeat(dequantize_scales(code2, c1), 64).astype(np.float64)
    cb = np.repeat(np.abs(x).reshape(-1, 64).max(axis=1), 64).astype(np.float64)
    bound = cb * (max_half_gap() + 2.0 ** -24) + np.abs(cb - a) + np.abs(w) * 2.0 ** -8 + a * 2.0 ** -23
    assert np.all(np.abs(x - w) <= bound)


def test_bits_per_parameter_closed_form():
    with open(os.path.join(GOLDEN, "double_quant_overhead.json")) as f:
        g = json.load(f)
    n = 4096 * 4096
    bpp = bits_per_parameter(n)
    assert bpp == 4.0 + g["bits_per_param_constants_after"]
    saving = g["bits_per_param_constants_before"] - (bpp - 4.0)
    assert abs(saving - g["pages_saving_bits_per_param"]) < 0.005
    gb = saving * g["pages_model_params"] / 8 / 1e9
    assert abs(gb - g["pages_saving_gb"]) < 0.05
    # The stored buffers of the oracle have exactly the sizes behind bpp.
    x = np.zeros(n, np.float32)
    packed, code2, c1 = quantize_nf4(x[: 64 * 256 * 4])
    assert packed.size == 64 * 256 * 4 // 2 and code2.size == 256 * 4 and c1.size == 4


def test_dequantize_at_equals_full_path():
    rng = np.random.default_rng(21)
    n = 64 * 256 * 5 + 100
    x = bf16_values(rng, n, 0.03)
    x[64 * 300:64 * 301] = 0.0
    packed, code2, c1 = quantize_nf4(x)
    full = dequantize_nf4(packed, code2, c1, n)
    idx = np.concatenate([rng.choice(n, 3000, replace=False), [0, n - 1, 64 * 300 + 5]])
    np.testing.assert_array_equal(dequantize_at(x, idx).view(np.uint32), full[idx].view(np.uint32))
