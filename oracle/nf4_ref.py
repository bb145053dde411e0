"""Oracle for the NF4 codec: codebook, blockwise quantization, double
quantization of the constants, dequantization to BFloat16.

TEST INFRASTRUCTURE ONLY (see the package header).  numpy, float64, every
rounding written out.

What the pages fix, and the readings taken where they are silent:

* "AI Glossary: QLoRA", second paragraph, and "QLoRA: Fine-Tuning 65-Billion
  Parameter Models ...", section "1. 4-bit NormalFloat (NF4)": NF4 is a 4-bit
  type for normally distributed values, built so that each quantization bucket
  gets the same share of values.  The pages print no values.  Reading: the
  levels are standard-normal quantiles at evenly spaced probabilities, taken
  separately for the positive side (8 levels) and the negative side (7
  levels), plus an exact zero, normalised to [-1, 1]; the outermost
  probability is delta = 1 - (1/30 + 1/32)/2.  Parity of the numbers beyond
  this construction: unpinned by the pages (they print none).
* Same two passages: the frozen weights are stored as 4-bit numbers with
  scaling constants.  Reading: absmax scaling over blocks of 64 consecutive
  elements of the row-major flattened weight; nearest level of the scaled
  value rounded to float32; ties to the lower index; an all-zero block gets
  the zero level (index 7); two codes per byte, first element in the high
  nibble.
* "AI Glossary: QLoRA", second paragraph, and "2. Double Quantization": the
  constants (float32) are themselves quantized.  Reading: blocks of 256
  constants, each scaled by the block's maximum (kept in float32) and coded
  with an unsigned linear 8-bit code k/255, nearest level, ties to the lower
  index, code 0 when the maximum is 0.
* "AI Glossary: QLoRA", second paragraph, and "QLoRA's Working Process":
  the 4-bit weights are turned back into BFloat16 each time the layer is
  used.  Reading: a' = fp32(fp32(k/255) * c1); w' = bf16(fp32(q_code * a')),
  each product a single correctly rounded float32 multiply, bf16 by
  round-to-nearest-even.
* "1. 4-bit NormalFloat (NF4)" names the usual 4-bit alternatives, Integer
  4-bit and Float 4-bit, and claims NF4 has the lower quantization error
  ("Performance and Evaluation", "NF4 efficiency"; the glossary's third
  paragraph: a plain 4-bit float scored about a point lower).  Neither format
  is defined on the pages.  Readings, both with the same block scaling,
  packing and double quantization as NF4, so only the 16 levels change:
    FP4  the 4-bit float with 1 sign, 2 exponent and 1 mantissa bit (bias 1,
         subnormals at exponent 0): magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6,
         divided by the largest, 6, so that the block absmax maps to +-1;
    Int4 the symmetric absmax integer code k/7, k = -7 .. 7.
  Each has 15 distinct values (FP4's +0 and -0 coincide); sorted, they fill
  indices 0..14 with the zero at index 7, and index 15 repeats the top level
  +1.  Ties go to the lower index, so code 15 is never produced and every
  code's value is the index's level, as for NF4.
* "2. Double Quantization" says only that the constants are quantized.  A
  second reading (``dq="centred_fp8"``; the original QLoRA paper's variant,
  not printed on the pages) codes them with an 8-bit float after removing
  their mean, since the constants are all positive:
    mu  = fp32(exact mean of all block absmaxes c_b of the tensor)
    d_b = fp32(c_b - mu)
    s_g = fp32(max |d_b| over the 256-group / 448)       (448: E4M3's largest)
    k_b = the E4M3 code (1 sign, 4 exponent bits with bias 7, 3 mantissa
          bits; no infinities) nearest to fp32(d_b / s_g), ties to the even
          code, saturating at +-448; a negative value that rounds to zero
          gives -0 (code 0x80); k_b = 0 when s_g = 0
    a'  = fp32(fp32(E4M3(k_b) * s_g) + mu)
  Stored: k_b in absmax_q, s_g per group in absmax_scale, then mu as one
  extra float at the end (NB2 + 1 floats).  Level 1 still uses the true c_b.
"""

from __future__ import annotations

from statistics import NormalDist

import numpy as np

BLOCK = 64  # elements per absmax block
GROUP = 256  # absmax constants per double-quantization block
ZERO_CODE = 7  # index of the exact-zero level


def nf4_codebook() -> np.ndarray:
    """The 16 NF4 levels as float32, sorted ascending.

    Quantile construction described in the module header ("1. 4-bit
    NormalFloat (NF4)": equal share of values per bucket for normal data).
    Built in float64 with the standard-library normal quantile, normalised by
    the largest level, then rounded once to float32.
    """
    inv = NormalDist().inv_cdf
    delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    pos_p = np.linspace(delta, 0.5, 9)[:-1]  # 8 probabilities, 0.5 excluded
    neg_p = np.linspace(delta, 0.5, 8)[:-1]  # 7 probabilities, 0.5 excluded
    pos = [inv(p) for p in pos_p]
    neg = [-inv(p) for p in neg_p]
    levels = np.array(sorted(pos + neg + [0.0]), dtype=np.float64)
    levels = levels / levels.max()
    return levels.astype(np.float32)


def fp4_codebook() -> np.ndarray:
    """The FP4 (1-2-1 float) levels as float32, sorted, divided by 6; index
    15 repeats +1 (see the module header)."""
    mags = []
    for m in range(8):  # 2 exponent bits, 1 mantissa bit
        e, f = m >> 1, m & 1
        mags.append(f * 0.5 if e == 0 else (1.0 + 0.5 * f) * 2.0 ** (e - 1))
    vals = sorted({v * sgn for v in mags for sgn in (1.0, -1.0)})  # 15 distinct (+-0 coincide)
    vals = np.array(vals + [max(vals)], dtype=np.float64) / max(mags)
    return vals.astype(np.float32)


def int4_codebook() -> np.ndarray:
    """The symmetric Int4 levels k/7, k = -7..7, as float32; index 15
    repeats +1 (see the module header)."""
    k = np.concatenate([np.arange(-7, 8), [7]]).astype(np.float64)
    return (k / 7.0).astype(np.float32)


CODEBOOKS = {"nf4": nf4_codebook, "fp4": fp4_codebook, "int4": int4_codebook}


def codebook(name: str = "nf4") -> np.ndarray:
    """The 16 float32 levels of the named 4-bit code ("nf4", "fp4", "int4")."""
    return CODEBOOKS[name]()


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16, ties to even.

    Returns float32 values that lie on the bfloat16 grid.  Finite inputs only.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    bits = (bits + 0x7FFF + lsb) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that already lie on the bf16 grid."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _nearest_index(values: np.ndarray, levels: np.ndarray, chunk: int = 1 << 20) -> np.ndarray:
    """argmin_i |values - levels[i]| in float64, first (lowest) index on ties.

    Evaluated in slices of ``chunk`` values only to bound memory."""
    lv = levels.astype(np.float64)[None, :]
    out = np.empty(values.size, dtype=np.int64)
    for s in range(0, values.size, chunk):
        d = np.abs(values[s:s + chunk].astype(np.float64)[:, None] - lv)
        out[s:s + chunk] = np.argmin(d, axis=1)
    return out


def _level2_table() -> np.ndarray:
    """fp32(k / 255) for k = 0..255 (the 8-bit constant code's levels)."""
    return (np.arange(256, dtype=np.float64) / 255.0).astype(np.float32)


def e4m3_value(code: int) -> float:
    """Value of an 8-bit E4M3 code (NaN for the two NaN codes)."""
    sign = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code of each float32 value, ties to the even code,
    saturating at +-448; the sign of a negative value is kept (-0 = 0x80)."""
    mags = np.array([e4m3_value(k) for k in range(0x7F)], dtype=np.float64)  # codes 0..126, ascending
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    a = np.minimum(np.abs(x), 448.0)
    hi = np.searchsorted(mags, a, side="left")          # first level >= a
    hi = np.minimum(hi, len(mags) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - mags[lo], mags[hi] - a
    code = np.where(dhi < dlo, hi, lo)
    tie = (dhi == dlo) & (hi != lo)
    code = np.where(tie, np.where(lo % 2 == 0, lo, hi), code)
    code = np.where(a == mags[hi], hi, code)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def _rn_f32_ratio(num: int, den: int) -> np.float32:
    """float32 nearest (ties to even) to the non-negative rational num/den."""
    if num == 0:
        return np.float32(0.0)
    # exponent e with 2^e <= num/den < 2^(e+1)
    e = num.bit_length() - den.bit_length()
    if (num << max(0, -e)) < (den << max(0, e)):
        e -= 1
    q = max(e, -126) - 23  # quantum of the result's binade (subnormals at 2^-149)
    if q >= 0:
        n, d = num, den << q
    else:
        n, d = num << -q, den
    m, r = divmod(n, d)
    if 2 * r > d or (2 * r == d and m % 2 == 1):
        m += 1
    return np.float32(m * 2.0 ** q)


def centred_mean(c: np.ndarray) -> np.float32:
    """fp32 of the exact mean of the block absmaxes (each a bf16 value)."""
    ints = (np.asarray(c, dtype=np.float64) * 2.0 ** 133)  # exact integers: bf16 values are multiples of 2^-133
    total = sum(int(v) for v in ints.tolist())
    return _rn_f32_ratio(total, len(ints) << 133)


def quantize_nf4(w: np.ndarray, block: int = BLOCK, group: int = GROUP, code: str = "nf4", dq: str = "linear8"):
    """Blockwise NF4 quantization with double-quantized constants (or the
    same scheme with the FP4 or Int4 levels, ``code`` = "fp4" / "int4"; the
    constants coded as in the module header, ``dq`` = "linear8" or
    "centred_fp8").

    ``w``: any-shape array of bfloat16 values (given as float32/float64 that
    lie on the bf16 grid), flattened row-major.

    Returns ``(codes, absmax_q, absmax_scale)``:
      codes        uint8[ceil(numel/2)]   two 4-bit codes per byte, first in
                                          the high nibble; a missing last
                                          element is padded with code 7
      absmax_q     uint8[NB]              8-bit code of each block's absmax
      absmax_scale float32[NB2]           the max absmax of each 256-group

    NB = ceil(numel/64), NB2 = ceil(NB/256).  A partial last block takes its
    absmax over the elements present; a partial last group its maximum over
    the constants present.
    """
    x = np.asarray(w, dtype=np.float32).reshape(-1)
    n = x.size
    nb = -(-n // block)
    q = codebook(code)

    # Level 1: per-block absmax c_b over the elements present.
    padded = np.zeros(nb * block, dtype=np.float32)
    padded[:n] = x
    present = np.zeros(nb * block, dtype=bool)
    present[:n] = True
    mag = np.where(present, np.abs(padded), 0.0).reshape(nb, block)
    c = mag.max(axis=1).astype(np.float32)  # exact: a bf16 value

    # Normalise: n = fp32(x / c_b) (the float64 quotient of two float32
    # values rounded to float32 equals the correctly rounded float32 quotient).
    cb = np.repeat(c, block)
    with np.errstate(invalid="ignore", divide="ignore"):
        normed = (padded.astype(np.float64) / cb.astype(np.float64)).astype(np.float32)
    normed = np.where(cb == 0, np.float32(0.0), normed)  # all-zero block -> level 7
    codes = _nearest_index(normed, q).astype(np.uint8)
    codes[~present] = ZERO_CODE

    # Pack two per byte: first element in the high nibble.
    if codes.size % 2:
        codes = np.concatenate([codes, np.array([ZERO_CODE], dtype=np.uint8)])
    pairs = codes.reshape(-1, 2)
    packed = ((pairs[:, 0] << 4) | pairs[:, 1]).astype(np.uint8)
    packed = packed[: (n + 1) // 2]

    nb2 = -(-nb // group)
    if dq == "centred_fp8":
        mu = centred_mean(c)
        d = (c.astype(np.float64) - np.float64(mu)).astype(np.float32)
        dpad = np.zeros(nb2 * group, dtype=np.float32)
        dpad[:nb] = np.abs(d)
        c1 = dpad.reshape(nb2, group).max(axis=1).astype(np.float32)
        sg = (c1.astype(np.float64) / 448.0).astype(np.float32)
        sb = np.repeat(sg, group)[:nb]
        with np.errstate(invalid="ignore", divide="ignore"):
            n2 = (d.astype(np.float64) / sb.astype(np.float64)).astype(np.float32)
        code2 = np.where(sb == 0, np.uint8(0), e4m3_encode(np.where(sb == 0, 0.0, n2))).astype(np.uint8)
        return packed, code2, np.concatenate([sg, [mu]]).astype(np.float32)
    if dq != "linear8":
        raise ValueError(dq)

    # Level 2: groups of 256 constants; c1 = max; code2 = nearest k/255 to
    # fp32(c_b / c1); code 0 when c1 == 0.
    cpad = np.zeros(nb2 * group, dtype=np.float32)
    cpad[:nb] = c
    c1 = cpad.reshape(nb2, group).max(axis=1).astype(np.float32)
    c1b = np.repeat(c1, group)[:nb]
    with np.errstate(invalid="ignore", divide="ignore"):
        n2 = (c.astype(np.float64) / c1b.astype(np.float64)).astype(np.float32)
    n2 = np.where(c1b == 0, np.float32(0.0), n2)
    code2 = _nearest_index(n2, _level2_table()).astype(np.uint8)
    return packed, code2, c1


def dequantize_scales(absmax_q: np.ndarray, absmax_scale: np.ndarray, group: int = GROUP,
                      dq: str = "linear8") -> np.ndarray:
    """Per-block dequantized constant a' = fp32(fp32(k/255) * c1), float32[NB]
    (``dq`` = "centred_fp8": a' = fp32(fp32(E4M3(k) * s_g) + mu))."""
    k = np.asarray(absmax_q, dtype=np.uint8)
    if dq == "centred_fp8":
        sc = np.asarray(absmax_scale, dtype=np.float32)
        mu = np.float64(sc[-1])
        v = np.array([e4m3_value(int(x)) for x in range(256)], dtype=np.float64)[k]
        sg = np.repeat(sc[:-1], group)[: k.size].astype(np.float64)
        p1 = (v * sg).astype(np.float32).astype(np.float64)  # exact product, one rounding
        return (p1 + mu).astype(np.float32)                   # exact sum, one rounding
    lvl = _level2_table()[k].astype(np.float64)
    c1 = np.repeat(np.asarray(absmax_scale, dtype=np.float32), group)[: k.size].astype(np.float64)
    return (lvl * c1).astype(np.float32)  # exact float64 product, one rounding


def dequantize_nf4(codes: np.ndarray, absmax_q: np.ndarray, absmax_scale: np.ndarray,
                   numel: int, block: int = BLOCK, group: int = GROUP, code: str = "nf4",
                   dq: str = "linear8") -> np.ndarray:
    """Dequantize to bfloat16 values (returned as float32 on the bf16 grid).

    w' = bf16(fp32(q_code * a')), a' from :func:`dequantize_scales`.
    """
    packed = np.asarray(codes, dtype=np.uint8)
    nib = np.empty(packed.size * 2, dtype=np.uint8)
    nib[0::2] = packed >> 4
    nib[1::2] = packed & 0xF
    nib = nib[:numel]
    q = codebook(code).astype(np.float64)
    a = dequantize_scales(absmax_q, absmax_scale, group, dq)
    ab = np.repeat(a, block)[:numel].astype(np.float64)
    w32 = (q[nib] * ab).astype(np.float32)  # exact float64 product, one rounding
    return bf16_round(w32)


def dequantize_at(w: np.ndarray, flat_idx: np.ndarray, block: int = BLOCK, group: int = GROUP,
                  code: str = "nf4") -> np.ndarray:
    """Quantize-then-dequantize only the elements at ``flat_idx`` of ``w``.

    Same definitions as :func:`quantize_nf4` followed by
    :func:`dequantize_nf4`, evaluated only where needed: every block absmax
    and group maximum is computed (they scale the requested elements), the
    nearest level and the bf16 product only for the requested elements.
    Used to check large layers on sampled outputs.
    """
    x = np.asarray(w, dtype=np.float32).reshape(-1)
    n = x.size
    nb = -(-n // block)
    padded = np.zeros(nb * block, dtype=np.float32)
    padded[:n] = x
    c = np.abs(padded).reshape(nb, block).max(axis=1).astype(np.float32)
    nb2 = -(-nb // group)
    cpad = np.zeros(nb2 * group, dtype=np.float32)
    cpad[:nb] = c
    c1 = cpad.reshape(nb2, group).max(axis=1).astype(np.float32)

    idx = np.asarray(flat_idx, dtype=np.int64).reshape(-1)
    b = idx // block
    cb = c[b]
    with np.errstate(invalid="ignore", divide="ignore"):
        normed = (x[idx].astype(np.float64) / cb.astype(np.float64)).astype(np.float32)
    normed = np.where(cb == 0, np.float32(0.0), normed)
    q = codebook(code)
    idx_code = _nearest_index(normed, q)
    c1b = c1[b // group]
    with np.errstate(invalid="ignore", divide="ignore"):
        n2 = (cb.astype(np.float64) / c1b.astype(np.float64)).astype(np.float32)
    n2 = np.where(c1b == 0, np.float32(0.0), n2)
    code2 = _nearest_index(n2, _level2_table())
    a = (_level2_table()[code2].astype(np.float64) * c1b.astype(np.float64)).astype(np.float32)
    w32 = (q.astype(np.float64)[idx_code] * a.astype(np.float64)).astype(np.float32)
    return bf16_round(w32)


def bits_per_parameter(numel: int, block: int = BLOCK, group: int = GROUP) -> float:
    """Stored bits per weight of the packed format (codes + both constant levels)."""
    nb = -(-numel // block)
    nb2 = -(-nb // group)
    return (8.0 * ((numel + 1) // 2) + 8.0 * nb + 32.0 * nb2) / numel


def max_half_gap(code: str = "nf4") -> float:
    """Largest distance from a value in [-1, 1] to its nearest level."""
    q = codebook(code).astype(np.float64)
    return float(np.max(np.diff(q)) / 2.0)


__all__ = [
    "BLOCK", "GROUP", "ZERO_CODE", "nf4_codebook", "fp4_codebook", "int4_codebook", "CODEBOOKS", "codebook",
    "bf16_round", "bf16_bits", "e4m3_value", "e4m3_encode", "centred_mean",
    "quantize_nf4", "dequantize_scales", "dequantize_nf4", "dequantize_at", "bits_per_parameter",
    "max_half_gap",
]
