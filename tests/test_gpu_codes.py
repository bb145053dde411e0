"""The FP4 and Int4 codes the pages compare NF4 with ("1. 4-bit NormalFloat
(NF4)": Integer 4-bit and Float 4-bit), run through the same kernels with
their own levels: packed codes, constants and dequantized weights bit for bit
against the oracle (ragged sizes, zero blocks, every bf16 value of a block,
every block-constant mantissa), and the LoRA linear forward and backward
within 2e-2 * RMS of the float64 oracle on that code's dequantized weight,
for the large-M GEMMs and the small-M forward."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from oracle import dequantize_nf4, lora_linear_backward, lora_linear_forward, quantize_nf4
from tests.helpers import assert_close_rms, f32, f64, u8

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
CODES = ["fp4", "int4"]


def assert_codec_equal(w, code):
    p = q.qlora_quantize_nf4(w.to(DEV), code=code)
    codes, aq, sc = quantize_nf4(f32(w), code=code)
    np.testing.assert_array_equal(u8(p.codes), codes)
    np.testing.assert_array_equal(u8(p.absmax_q), aq)
    np.testing.assert_array_equal(p.absmax_scale.cpu().numpy(), sc)
    ref = dequantize_nf4(codes, aq, sc, w.numel(), code=code)
    got = f32(q.qlora_dequantize_nf4(p)).reshape(-1)
    np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))
    nib = np.concatenate([codes >> 4, codes & 15])
    assert not np.any(nib == 15)
    return p


@pytest.mark.parametrize("code", CODES)
@pytest.mark.parametrize("n", [1, 65, 16384 + 5, 3 * 16384 + 100])
def test_ragged_sizes(code, n):
    x = np.random.default_rng(n).standard_normal(n).astype(np.float32) * 0.02
    if n > 200:
        x[64:192] = 0.0
        x[5] = 3.0
    assert_codec_equal(synthetic.to_bf16(x), code)


@pytest.mark.parametrize("code", CODES)
def test_every_bf16_pattern(code):
    bits = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    allv = bits[np.isfinite(bits)]
    for c in (1.0, 0.0234375, 7.0e4, 1.5e-38):
        c = float(synthetic.to_bf16(np.array([c], np.float32)).float()[0])
        xs = allv[np.abs(allv) <= c]
        blocks = np.repeat(xs[:, None], 64, axis=1)
        blocks[:, 0] = c
        assert_codec_equal(synthetic.to_bf16(blocks.reshape(-1)), code)


@pytest.mark.parametrize("code", CODES)
def test_every_block_constant_mantissa(code):
    bits = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    base = bits[np.isfinite(bits) & (np.abs(bits) >= 2.0 ** -10) & (np.abs(bits) < 2.0)]
    blocks = []
    for scale in (1.0, 2.0 ** 100, 2.0 ** 127):
        for m in range(128):
            c = np.float32((1.0 + m / 128.0) * scale)
            xs = base[np.abs(base) <= 1.0 + m / 128.0].astype(np.float64) * scale
            xs = np.concatenate([xs, np.zeros((-len(xs)) % 63)]).astype(np.float32).reshape(-1, 63)
            blocks.append(np.concatenate([np.full((len(xs), 1), c, np.float32), xs], axis=1))
    assert_codec_equal(synthetic.to_bf16(np.concatenate(blocks).reshape(-1)), code)


@pytest.mark.parametrize("code", CODES)
@pytest.mark.parametrize("M,K,N,r", [(600, 512, 776, 16), (16, 4096, 1024, 64)])
def test_linear_forward_backward(code, M, K, N, r):
    case = synthetic.linear_case(M, K, N, r, 0.5, seed=M + N + len(code))
    p = assert_codec_equal(case.W, code)
    X, A, B, dY = (t.to(DEV) for t in (case.X, case.A, case.B, case.dY))
    ws = q.new_workspace(M, K, N, r, DEV)
    Y, T = q.qlora_linear_fwd(X, p, A, B, case.scale, workspace=ws)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, T, p, A, B, case.scale, workspace=ws)
    assert q.qlora_check_status(ws) == 0
    codes, aq, sc = quantize_nf4(f32(case.W), code=code)
    Wdq = dequantize_nf4(codes, aq, sc, case.W.numel(), code=code).reshape(N, K)
    Yr, Tr = lora_linear_forward(f64(case.X), Wdq, f64(case.A), f64(case.B), case.scale)
    dXr, dAr, dBr = lora_linear_backward(f64(case.dY), f64(case.X), Wdq, f64(case.A), f64(case.B), case.scale)
    for name, got, ref in (("Y", Y, Yr), ("T", T, Tr), ("dX", dX, dXr), ("dA", dA, dAr), ("dB", dB, dBr)):
        assert_close_rms(f64(got), ref, f"{code} {name}")


def test_nf4_has_the_lowest_error_on_the_gpu_too():
    """The pages' comparison, on the library's own quantize + dequantize of
    a LLaMA-shaped N(0, 0.02^2) weight."""
    W = synthetic.weight_only(4096, 4096, seed=17).to(DEV)
    err = {}
    for code in ("nf4", "fp4", "int4"):
        Wd = q.qlora_dequantize_nf4(q.qlora_quantize_nf4(W, code=code))
        err[code] = float(((Wd.double() - W.double()) ** 2).mean())
    assert err["nf4"] < err["fp4"] and err["nf4"] < err["int4"], err
