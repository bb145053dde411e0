"""GPU parity of the LoRA linear forward and backward against the float64
oracle (same dequantized weight): max abs error <= 2e-2 * RMS(oracle) for
Y, T, dX, dA, dB; exact special cases."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from oracle import quantize_nf4, dequantize_nf4, lora_linear_forward, lora_linear_backward
from tests.helpers import assert_close_rms, f32, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run_gpu(case):
    Wp = q.qlora_quantize_nf4(case.W.to(DEV))
    X, A, B, dY = (t.to(DEV) for t in (case.X, case.A, case.B, case.dY))
    ws = q.new_workspace(case.M, case.K, case.N, case.r, DEV)
    Y, T = q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, T, Wp, A, B, case.scale, workspace=ws)
    assert q.qlora_check_status(ws) == 0
    return dict(Y=Y, T=T, dX=dX, dA=dA, dB=dB, Wp=Wp)


def oracle_wdq(case):
    codes, aq, sc = quantize_nf4(f32(case.W))
    return dequantize_nf4(codes, aq, sc, case.W.numel()).reshape(case.N, case.K)


def check_full(case, g, Wdq=None):
    Wdq = oracle_wdq(case) if Wdq is None else Wdq
    X, A, B, dY = f64(case.X), f64(case.A), f64(case.B), f64(case.dY)
    Y, T = lora_linear_forward(X, Wdq, A, B, case.scale)
    dX, dA, dB = lora_linear_backward(dY, X, Wdq, A, B, case.scale)
    errs = {}
    for name, ref in (("Y", Y), ("T", T), ("dX", dX), ("dA", dA), ("dB", dB)):
        errs[name] = assert_close_rms(f64(g[name]), ref, name)
    return errs


def test_tiny_layer():
    """256 x 256 weight, 16 tokens, r = 8, scale 2 (seed 0)."""
    case = synthetic.tiny_case()
    check_full(case, run_gpu(case))


@pytest.mark.parametrize("M,K,N,r", [(200, 320, 264, 16), (129, 64, 8, 8), (300, 576, 520, 72),
                                     (1, 256, 256, 64), (77, 1024, 1000, 128), (16, 8192, 256, 64)])
def test_ragged_shapes(M, K, N, r):
    case = synthetic.linear_case(M, K, N, r, 0.5, seed=M + K + N + r)
    check_full(case, run_gpu(case))


# Forward shapes of the weight-streaming path (M <= 128 tokens): every token
# padding width (16, 32, 64, 128), ragged weight tiles (N % 128 != 0), one
# reduction block (K = 64), LoRA ranks with one or two 64-column blocks, and
# products whose 128-row tiles are split over several CTAs.
@pytest.mark.parametrize("M,K,N,r", [(2, 64, 136, 8), (17, 4096, 1024, 64), (33, 1536, 1000, 72),
                                     (64, 2048, 2056, 128), (65, 640, 392, 16), (128, 4096, 776, 64),
                                     (8, 11008, 512, 64)])
def test_small_m_shapes(M, K, N, r):
    case = synthetic.linear_case(M, K, N, r, 0.5, seed=3 * M + K + N + r)
    check_full(case, run_gpu(case))


def test_small_m_repeated_calls_are_identical():
    """Split tiles are summed through per-tile counters that each call resets:
    three calls on one workspace give the same bits."""
    case = synthetic.linear_case(16, 4096, 2048, 64, 0.25, seed=19)
    Wp = q.qlora_quantize_nf4(case.W.to(DEV))
    X, A, B = (t.to(DEV) for t in (case.X, case.A, case.B))
    ws = q.new_workspace(case.M, case.K, case.N, case.r, DEV)
    outs = [q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws)[0] for _ in range(3)]
    assert q.qlora_check_status(ws) == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    Wdq = oracle_wdq(case)
    Y, _ = lora_linear_forward(f64(case.X), Wdq, f64(case.A), f64(case.B), case.scale)
    assert_close_rms(f64(outs[0]), Y, "Y")


def test_repeated_calls_on_one_workspace_are_identical():
    """The GEMM launches hand out work by ticket and publish T and U per
    512-row block through counters in the workspace that each launch returns
    to zero: three forward + backward passes on one workspace give the same
    bits (a counter left behind would stall the next call into a timeout)."""
    case = synthetic.linear_case(1100, 512, 640, 64, 0.25, seed=31)
    Wp = q.qlora_quantize_nf4(case.W.to(DEV))
    X, A, B, dY = (t.to(DEV) for t in (case.X, case.A, case.B, case.dY))
    ws = q.new_workspace(case.M, case.K, case.N, case.r, DEV)
    runs = []
    for _ in range(3):
        Y, T = q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws)
        runs.append((Y, T) + tuple(q.qlora_linear_bwd(dY, X, T, Wp, A, B, case.scale, workspace=ws)))
    assert q.qlora_check_status(ws) == 0
    for k in range(5):
        assert torch.equal(runs[0][k], runs[1][k]) and torch.equal(runs[0][k], runs[2][k]), k
    check_full(case, dict(zip(("Y", "T", "dX", "dA", "dB"), runs[0])))


def test_many_row_blocks_few_column_tiles():
    """16 row blocks and one column tile: as many rank units as output tiles."""
    case = synthetic.linear_case(8000, 256, 200, 72, 0.5, seed=33)
    check_full(case, run_gpu(case))


def test_special_cases_exact():
    base = synthetic.linear_case(192, 256, 320, 16, 1.0, seed=21)
    # B = 0: no gradient reaches A, bit-exactly; Y is the frozen product.
    zb = synthetic.LinearCase(base.W, base.X, base.A, torch.zeros_like(base.B), base.dY, 1.0)
    g = run_gpu(zb)
    assert torch.count_nonzero(g["dA"]) == 0
    check_full(zb, g)
    # A = 0: T = 0 and dB = 0 exactly.
    za = synthetic.LinearCase(base.W, base.X, torch.zeros_like(base.A), base.B, base.dY, 1.0)
    g = run_gpu(za)
    assert torch.count_nonzero(g["T"]) == 0 and torch.count_nonzero(g["dB"]) == 0
    # s = 0: the dense layer.
    s0 = synthetic.LinearCase(base.W, base.X, base.A, base.B, base.dY, 0.0)
    g = run_gpu(s0)
    assert torch.count_nonzero(g["T"]) == 0 and torch.count_nonzero(g["dA"]) == 0
    check_full(s0, g)


def test_dense_product_matches_torch_on_dequantized_weight():
    """With s = 0, Y equals a library bf16 matmul of X and the dequantized W."""
    case = synthetic.linear_case(512, 1024, 768, 16, 0.0, seed=5)
    g = run_gpu(case)
    Wd = q.qlora_dequantize_nf4(g["Wp"])
    ref = (case.X.to(DEV).float() @ Wd.float().t())
    assert_close_rms(f64(g["Y"]), ref.double().cpu().numpy(), "Y vs torch")


def test_backward_is_bit_reproducible():
    case = synthetic.linear_case(1024, 512, 640, 64, 0.25, seed=8)
    g1, g2 = run_gpu(case), run_gpu(case)
    for k in ("Y", "T", "dX", "dA", "dB"):
        assert torch.equal(g1[k], g2[k]), k


def test_attention_projection_full_size_sampled_rows():
    """LLaMA-7B attention projection (4096^2, 4096 tokens, r = 64, scale 0.25):
    Y and dX checked on 512 seeded rows (a row of a row-wise product depends
    only on that row), T, dA and dB in full."""
    case = synthetic.attn_proj_case()
    g = run_gpu(case)
    Wdq = oracle_wdq(case)
    rows = np.sort(np.random.default_rng(123).choice(case.M, 512, replace=False))
    X, A, B, dY = f64(case.X), f64(case.A), f64(case.B), f64(case.dY)
    Yr, _ = lora_linear_forward(X[rows], Wdq, A, B, case.scale)
    assert_close_rms(f64(g["Y"])[rows], Yr, "Y rows")
    T = case.scale * (X @ A)
    assert_close_rms(f64(g["T"]), T, "T")
    dXr, _, _ = lora_linear_backward(dY[rows], X[rows], Wdq, A, B, case.scale)
    assert_close_rms(f64(g["dX"])[rows], dXr, "dX rows")
    U = case.scale * (dY @ B.T)
    assert_close_rms(f64(g["dA"]), X.T @ U, "dA")
    assert_close_rms(f64(g["dB"]), case.scale * (X @ A).T @ dY, "dB")


# Any rank 1 <= r <= 256: multiples of 8 up to 128 run as they are, others
# with the adapter padded to a multiple of 8 in the workspace, and ranks above
# 128 with the rank units taking 128 adapter columns per CTA and the dA / dB
# units split into column chunks.  Large-M (pair GEMMs) and small-M shapes.
@pytest.mark.parametrize("M,K,N,r", [(600, 512, 776, 4), (600, 512, 776, 200), (300, 320, 264, 1),
                                     (700, 640, 392, 13), (520, 576, 520, 136), (600, 512, 256, 192),
                                     (1100, 512, 640, 256), (16, 4096, 1024, 4), (16, 2048, 1000, 200),
                                     (64, 1024, 512, 77), (1, 256, 256, 256)])
def test_any_rank(M, K, N, r):
    case = synthetic.linear_case(M, K, N, r, 0.5, seed=M + K + N + r)
    check_full(case, run_gpu(case))


# One token (M = 1): ragged row counts and depths, every rank path.
@pytest.mark.parametrize("K,N,r", [(64, 8, 8), (1024, 1000, 64), (16384, 136, 16), (4096, 4104, 5),
                                   (8192, 1024, 256), (16448, 264, 64)])
def test_single_token(K, N, r):
    case = synthetic.linear_case(1, K, N, r, 0.5, seed=K + N + r)
    check_full(case, run_gpu(case))


def test_single_token_is_bit_reproducible():
    case = synthetic.linear_case(1, 8192, 2056, 64, 0.25, seed=44)
    g1, g2 = run_gpu(case), run_gpu(case)
    assert torch.equal(g1["Y"], g2["Y"]) and torch.equal(g1["T"], g2["T"])
