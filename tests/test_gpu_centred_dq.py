"""The mean-centred 8-bit-float double quantization (the second reading of
"2. Double Quantization"; QLORA_DQ_CENTRED_FP8) on the GPU: packed codes,
E4M3 constant codes, group scales and the exact mean bit for bit against the
oracle, for each 4-bit code, on ragged sizes, zero blocks, outliers, wide
exponent ranges and a full LLaMA-7B projection; the dequantized weight bit
for bit; and the linear layer's forward and backward within 2e-2 * RMS of
the float64 oracle on that weight (large-M GEMMs and the small-M forward)."""

import numpy as np
import pytest

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from oracle import dequantize_nf4, lora_linear_backward, lora_linear_forward, quantize_nf4
from tests.helpers import assert_close_rms, f32, f64, u8

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
DQ = "centred_fp8"


def assert_codec_equal(w, code="nf4"):
    p = q.qlora_quantize_nf4(w.to(DEV), code=code, dq=DQ)
    codes, aq, sc = quantize_nf4(f32(w), code=code, dq=DQ)
    np.testing.assert_array_equal(p.absmax_scale.cpu().numpy().view(np.uint32), sc.view(np.uint32))
    np.testing.assert_array_equal(u8(p.absmax_q), aq)
    np.testing.assert_array_equal(u8(p.codes), codes)
    ref = dequantize_nf4(codes, aq, sc, w.numel(), code=code, dq=DQ)
    got = f32(q.qlora_dequantize_nf4(p)).reshape(-1)
    np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert q.qlora_check_status(None) == 0
    return p


@pytest.mark.parametrize("code", ["nf4", "fp4", "int4"])
@pytest.mark.parametrize("n", [1, 64, 65, 16384 + 5, 3 * 16384 + 100])
def test_ragged_sizes(code, n):
    x = np.random.default_rng(n + 7).standard_normal(n).astype(np.float32) * 0.02
    if n > 200:
        x[64:192] = 0.0
        x[5] = 3.0
    assert_codec_equal(synthetic.to_bf16(x), code)


def test_wide_exponent_range():
    """Block absmaxes from 1e-35 to 1e30 (the exact mean needs every bit)."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2000, 64)).astype(np.float32)
    x *= (10.0 ** rng.uniform(-35, 30, (2000, 1))).astype(np.float32)
    assert_codec_equal(synthetic.to_bf16(x.reshape(-1)))


def test_attention_projection_weight_full_size():
    assert_codec_equal(synthetic.attn_proj_case().W)


@pytest.mark.parametrize("M,K,N,r", [(600, 512, 776, 16), (16, 4096, 1024, 64)])
def test_linear_forward_backward(M, K, N, r):
    case = synthetic.linear_case(M, K, N, r, 0.5, seed=M + N + 5)
    p = assert_codec_equal(case.W)
    X, A, B, dY = (t.to(DEV) for t in (case.X, case.A, case.B, case.dY))
    ws = q.new_workspace(M, K, N, r, DEV)
    Y, T = q.qlora_linear_fwd(X, p, A, B, case.scale, workspace=ws)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, T, p, A, B, case.scale, workspace=ws)
    assert q.qlora_check_status(ws) == 0
    codes, aq, sc = quantize_nf4(f32(case.W), dq=DQ)
    Wdq = dequantize_nf4(codes, aq, sc, case.W.numel(), dq=DQ).reshape(N, K)
    Yr, Tr = lora_linear_forward(f64(case.X), Wdq, f64(case.A), f64(case.B), case.scale)
    dXr, dAr, dBr = lora_linear_backward(f64(case.dY), f64(case.X), Wdq, f64(case.A), f64(case.B), case.scale)
    for name, got, ref in (("Y", Y, Yr), ("T", T, Tr), ("dX", dX, dXr), ("dA", dA, dAr), ("dB", dB, dBr)):
        assert_close_rms(f64(got), ref, name)
