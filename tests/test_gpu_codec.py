"""GPU parity of the NF4 codec: packed codes, quantized constants and
dequantized bf16 weights must equal the oracle bit for bit."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from oracle import quantize_nf4, dequantize_nf4
from tests.helpers import f32, u8

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def gpu_quantize(w_cpu_bf16):
    return q.qlora_quantize_nf4(w_cpu_bf16.to(DEV))


def assert_codec_equal(w_cpu_bf16):
    p = gpu_quantize(w_cpu_bf16)
    codes, aq, sc = quantize_nf4(f32(w_cpu_bf16))
    np.testing.assert_array_equal(u8(p.codes), codes)
    np.testing.assert_array_equal(u8(p.absmax_q), aq)
    np.testing.assert_array_equal(p.absmax_scale.cpu().numpy(), sc)
    deq = q.qlora_dequantize_nf4(p)
    ref = dequantize_nf4(codes, aq, sc, w_cpu_bf16.numel())
    np.testing.assert_array_equal(f32(deq).reshape(-1).view(np.uint32), ref.view(np.uint32))
    return p


def test_tiny_layer_weight():
    assert_codec_equal(synthetic.tiny_case().W)


@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 1000, 16384, 16384 + 5, 3 * 16384 + 100, 64 * 257])
def test_ragged_sizes(n):
    w = synthetic.to_bf16(np.random.default_rng(n).standard_normal(n).astype(np.float32) * 0.02)
    assert_codec_equal(w)


def test_zero_blocks_and_outliers():
    x = np.random.default_rng(9).standard_normal(64 * 600).astype(np.float32) * 0.02
    x[64 * 3:64 * 5] = 0.0              # zero blocks
    x[64 * 256:64 * 512] = 0.0           # a whole zero group
    x[7] = 5.0                           # outlier
    x[64 * 520 + 3] = -1e-30             # tiny magnitudes (subnormal bf16 region)
    assert_codec_equal(synthetic.to_bf16(x))


def test_every_bf16_pattern():
    bits = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    allv = bits[np.isfinite(bits)]
    for c in (1.0, 0.75, 0.0234375, 3.0, 7.0e4, 1.5e-38):
        c = float(synthetic.to_bf16(np.array([c], np.float32)).float()[0])
        xs = allv[np.abs(allv) <= c]
        blocks = np.repeat(xs[:, None], 64, axis=1)
        blocks[:, 0] = c
        assert_codec_equal(synthetic.to_bf16(blocks.reshape(-1)))


def test_every_block_constant_mantissa():
    """Thresholds of a block constant c = m * 2^e come from a per-mantissa
    table scaled by 2^e: every one of the 128 bf16 mantissas, at three
    exponents and next to the smallest exponent that uses the table, with
    every bf16 value of [-c, c] above c * 2^-10 spread over blocks whose
    first element is c (so c is each block's absmax)."""
    bits = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    base = bits[np.isfinite(bits) & (np.abs(bits) >= 2.0 ** -10) & (np.abs(bits) < 2.0)]
    blocks = []
    for scale in (1.0, 2.0 ** -100, 2.0 ** 100, 2.0 ** -121, 2.0 ** -122):
        for m in range(128):
            c = np.float32((1.0 + m / 128.0) * scale)
            xs = base[np.abs(base) <= 1.0 + m / 128.0].astype(np.float64) * scale
            xs = np.concatenate([xs, np.zeros((-len(xs)) % 63)]).astype(np.float32).reshape(-1, 63)
            blocks.append(np.concatenate([np.full((len(xs), 1), c, np.float32), xs], axis=1))
            if scale in (2.0 ** -121, 2.0 ** -122) and m >= 3:
                break
    assert_codec_equal(synthetic.to_bf16(np.concatenate(blocks).reshape(-1)))


def test_dequantize_arbitrary_packed_input():
    rng = np.random.default_rng(4)
    n = 64 * 256 * 3 + 64 * 7
    codes = rng.integers(0, 256, (n + 1) // 2, dtype=np.uint8)
    aq = rng.integers(0, 256, n // 64, dtype=np.uint8)
    sc = np.abs(rng.standard_normal(-(-(n // 64) // 256))).astype(np.float32)
    p = q.PackedNF4(torch.from_numpy(codes).to(DEV), torch.from_numpy(aq).to(DEV), torch.from_numpy(sc).to(DEV), (n,))
    got = f32(q.qlora_dequantize_nf4(p)).view(np.uint32)
    ref = dequantize_nf4(codes, aq, sc, n).view(np.uint32)
    np.testing.assert_array_equal(got, ref)


def test_attention_projection_weight_full_size():
    """LLaMA-7B attention projection, 4096 x 4096 with 0.1% x10 outliers."""
    assert_codec_equal(synthetic.attn_proj_case().W)


def test_quantize_is_deterministic():
    w = synthetic.weight_only(512, 4096, seed=12).to(DEV)
    a, b = q.qlora_quantize_nf4(w), q.qlora_quantize_nf4(w)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.absmax_q, b.absmax_q)
    assert torch.equal(a.absmax_scale, b.absmax_scale)
