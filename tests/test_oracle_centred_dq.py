"""Pins for the oracle's mean-centred 8-bit-float double quantization (the
reading of "2. Double Quantization" that codes the constants with E4M3 after
removing their mean; see oracle/nf4_ref.py).

* E4M3 values: closed forms (1 = 0x38, largest 448 = 0x7E, smallest
  subnormal 2^-9 = 0x01, NaN at 0x7F / 0xFF).
* E4M3 encoding: exact-rational nearest search with ties to the even code,
  and torch's own float32 -> float8_e4m3fn cast (a library route) on every
  in-range value tested.
* The mean: exact rational arithmetic (tests/exact.py), and special cases.
* The whole codec: element-by-element restatement in exact rationals on
  small and ragged sizes, plus special cases (a group of equal constants
  codes 0 and dequantizes to the mean exactly).
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import bf16_round, dequantize_nf4
from oracle.nf4_ref import (bits_per_parameter, centred_mean, dequantize_scales, e4m3_encode, e4m3_value,
                            nf4_codebook, quantize_nf4)
from tests.exact import frac, rn_bf16, rn_f32

E4M3 = {k: Fraction(e4m3_value(k)) for k in range(256) if k not in (0x7F, 0xFF)}


def test_e4m3_closed_forms():
    assert e4m3_value(0x38) == 1.0 and e4m3_value(0x7E) == 448.0 and e4m3_value(0xFE) == -448.0
    assert e4m3_value(0x01) == 2.0 ** -9 and e4m3_value(0x08) == 2.0 ** -6 and e4m3_value(0x07) == 7 * 2.0 ** -9
    assert np.isnan(e4m3_value(0x7F)) and np.isnan(e4m3_value(0xFF))
    assert e4m3_value(0x80) == 0.0 and np.signbit(e4m3_value(0x80))


def brute_e4m3(x: Fraction, negative: bool) -> int:
    a = min(abs(x), Fraction(448))
    best = None
    for k in range(0x7F):
        d = abs(E4M3[k] - a)
        if best is None or d < best[0] or (d == best[0] and k % 2 == 0):
            best = (d, k)
    return best[1] | (0x80 if negative else 0)


def test_e4m3_encode_brute_force_and_torch():
    rng = np.random.default_rng(3)
    vals = np.concatenate([
        rng.standard_normal(3000) * 50, rng.standard_normal(500) * 0.01, rng.uniform(-460, 460, 500),
        [0.0, -0.0, 448.0, -448.0, 449.0, 464.0, 1e6, -1e-12, 1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10],
    ]).astype(np.float32)
    got = e4m3_encode(vals)
    for v, g in zip(vals.tolist(), got.tolist()):
        assert g == brute_e4m3(Fraction(v), np.signbit(np.float32(v))), (v, hex(g))
    inr = np.abs(vals) <= 448
    t = torch.from_numpy(vals[inr]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got[inr], t)


def test_mean_is_the_exact_mean_rounded_once():
    rng = np.random.default_rng(9)
    for n in (1, 2, 3, 257, 10000):
        c = bf16_round(np.abs(rng.standard_normal(n)).astype(np.float32) * np.float32(10.0 ** rng.integers(-30, 30)))
        ref = rn_f32(sum(frac(v) for v in c) / n)
        assert frac(centred_mean(c)) == ref
    assert centred_mean(np.zeros(5, np.float32)) == 0.0
    assert centred_mean(np.full(7, 0.375, np.float32)) == np.float32(0.375)


def brute_centred(x, block=64, group=256):
    xs = [frac(v) for v in x]
    n = len(xs)
    nb = -(-n // block)
    c = [max(abs(v) for v in xs[b * block:(b + 1) * block]) for b in range(nb)]
    q = [frac(v) for v in nf4_codebook()]
    codes = []
    for i, v in enumerate(xs):
        cb = c[i // block]
        codes.append(7 if cb == 0 else min(range(16), key=lambda j: (abs(rn_f32(v / cb) - q[j]), j)))
    if n % 2:
        codes.append(7)
    packed = [codes[2 * j] * 16 + codes[2 * j + 1] for j in range(len(codes) // 2)]
    mu = rn_f32(sum(c) / nb)
    d = [rn_f32(cb - mu) for cb in c]
    nb2 = -(-nb // group)
    sg = [rn_f32(max(abs(v) for v in d[g * group:(g + 1) * group]) / 448) for g in range(nb2)]
    k = [0 if sg[b // group] == 0 else brute_e4m3(rn_f32(d[b] / sg[b // group]), d[b] < 0) for b in range(nb)]
    a = [rn_f32(rn_f32(E4M3[k[b]] * sg[b // group]) + mu) for b in range(nb)]
    nib = [v for byte in packed for v in (byte >> 4, byte & 15)]
    w = [rn_bf16(rn_f32(q[nib[i]] * a[i // block])) for i in range(n)]
    return packed, k, sg + [mu], w


@pytest.mark.parametrize("n", [64, 65, 64 * 256 + 100])
def test_codec_matches_brute_force(n):
    rng = np.random.default_rng(n)
    x = bf16_round(rng.standard_normal(n).astype(np.float32) * np.float32(0.02))
    if n > 1000:
        x[:64] = 0.0
        x[64 * 3] = 0.5
    packed, code2, sc = quantize_nf4(x, dq="centred_fp8")
    bp, bk, bsc, bw = brute_centred(list(x))
    assert packed.tolist() == bp
    assert code2.tolist() == bk
    assert [frac(v) for v in sc] == bsc
    w = dequantize_nf4(packed, code2, sc, n, dq="centred_fp8")
    assert [frac(v) for v in w] == bw


def test_equal_constants_dequantize_to_the_mean():
    x = np.zeros((300, 64), np.float32)
    x[:, 0] = 0.25  # every block absmax is 0.25
    x[:, 1:] = 0.01
    x = bf16_round(x.reshape(-1))
    packed, code2, sc = quantize_nf4(x, dq="centred_fp8")
    assert sc[-1] == np.float32(0.25) and np.all(sc[:-1] == 0) and np.all(code2 == 0)
    np.testing.assert_array_equal(dequantize_scales(code2, sc, dq="centred_fp8"), np.full(300, 0.25, np.float32))


def test_overhead_is_one_float_more():
    n = 4096 * 4096
    assert bits_per_parameter(n) == 4.0 + 8.0 / 64 + 32.0 / (64 * 256)
    _, code2, sc = quantize_nf4(np.zeros(64 * 256 * 2, np.float32), dq="centred_fp8")
    assert code2.size == 512 and sc.size == 3  # two group scales and the mean
