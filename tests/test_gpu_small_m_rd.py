"""GPU parity of the forward for few tokens on the path that decodes the
4-bit weight into register fragments of the tensor-core MMA and applies each
block constant to its block's partial product (M <= 8, and 9 <= M <= 16
for weights of 2^27 elements or more): Y and T within 2e-2 * RMS of the
float64 oracle on the same dequantized weight, over ragged inputs
(K % 256 != 0, K % 1024 != 0), ragged row blocks (N % 256 != 0), both token
widths of a fragment (8 and 16), ranks 1..128, every code and constant
scheme, and bit-identical repeated calls."""

import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from oracle import dequantize_nf4, lora_linear_forward, quantize_nf4
from tests.helpers import assert_close_rms, f32, f64
from tests.test_gpu_configs import check_linear_sampled, run_linear

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def forward(case, code="nf4", dq="linear8", ws=None):
    Wp = q.qlora_quantize_nf4(case.W.to(DEV), code=code, dq=dq)
    X, A, B = (t.to(DEV) for t in (case.X, case.A, case.B))
    ws = q.new_workspace(case.M, case.K, case.N, case.r, DEV) if ws is None else ws
    Y, T = q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws)
    assert q.qlora_check_status(ws) == 0
    return Y, T


def check(case, Y, T, code="nf4", dq="linear8"):
    codes, aq, sc = quantize_nf4(f32(case.W), code=code, dq=dq)
    Wdq = dequantize_nf4(codes, aq, sc, case.W.numel(), code=code, dq=dq).reshape(case.N, case.K)
    Yr, Tr = lora_linear_forward(f64(case.X), Wdq, f64(case.A), f64(case.B), case.scale)
    assert_close_rms(f64(Y), Yr, "Y")
    assert_close_rms(f64(T), Tr, "T")


# (M, K, N, r): one block and one chunk; a last chunk with one block
# (K % 256 == 64); 4-byte but not 16-byte constant rows (K % 1024 != 0);
# 8-row and 264-row weights (row blocks cut by N); every token count class.
SHAPES = [(1, 64, 8, 1), (3, 192, 264, 4), (8, 320, 520, 16), (2, 1088, 1000, 72), (7, 2048, 2056, 128),
          (5, 4160, 776, 64), (4, 3072, 4104, 8), (8, 8192, 1536, 64), (1, 11008, 4096, 64)]


@pytest.mark.parametrize("M,K,N,r", SHAPES)
def test_shapes(M, K, N, r):
    case = synthetic.linear_case(M, K, N, r, 0.25, seed=7 * M + K + N + r, outlier_frac=0.001)
    Y, T = forward(case)
    check(case, Y, T)


# 9..16 tokens (16-wide fragments) take this path for weights of 2^27
# elements or more: Y checked on sampled output columns, T in full.
@pytest.mark.parametrize("M,K,N,r", [(16, 8192, 16384, 64), (12, 4160, 32264, 8)])
def test_sixteen_wide(M, K, N, r):
    case = synthetic.linear_case(M, K, N, r, 0.25, seed=M + K + N + r, with_dy=False)
    g = run_linear(case, backward=False)
    check_linear_sampled(case, g, seed=M + N, backward=False, n_rows=M, n_cols=256)


@pytest.mark.parametrize("code", ["nf4", "fp4", "int4"])
@pytest.mark.parametrize("dq", ["linear8", "centred_fp8"])
def test_codes(code, dq):
    case = synthetic.linear_case(6, 2112, 520, 24, 0.5, seed=101)
    Y, T = forward(case, code, dq)
    check(case, Y, T, code, dq)


def test_repeated_calls_are_identical():
    """Row blocks split over CTAs are summed by the last of their warps in a
    fixed order through per-row-group counters that each call returns to
    zero: repeated calls on one workspace give the same bits."""
    case = synthetic.linear_case(8, 4096, 3072, 64, 0.25, seed=23)
    ws = q.new_workspace(case.M, case.K, case.N, case.r, DEV)
    outs = [forward(case, ws=ws) for _ in range(3)]
    for Y, T in outs[1:]:
        assert torch.equal(Y, outs[0][0]) and torch.equal(T, outs[0][1])
    check(case, *outs[0])
