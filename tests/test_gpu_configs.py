"""GPU parity at the full workload sizes: the LLaMA-7B MLP trio (SiLU-gated),
the seven LLaMA-65B-shaped linears (with the one-shot quantization of their
weights) and the small-M forward sweep.

Full-size float64 products are out of reach on the host, so the checks use
properties that hold at any size:
  * Y and dX on sampled (row, column) entries: an entry of a matrix product
    depends only on one row and one column, and the oracle dequantizes just
    the weight elements those entries need (every block absmax and group
    maximum is still computed);
  * T, dA and dB in full (rank-r products, cheap in float64);
  * packed codes and constants bit-exact on sampled 256-block groups (each
    group is quantized independently).
Tolerance as everywhere: max abs error <= 2e-2 * RMS of the float64 oracle.
"""

import numpy as np
import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from oracle import dequantize_at, quantize_nf4
from tests.helpers import assert_close_rms, f32, f64, u8

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def oracle_rows(W, rows):
    """Dequantized rows `rows` of W [N, K] (float64)."""
    N, K = W.shape
    idx = (np.asarray(rows)[:, None] * K + np.arange(K)[None, :]).reshape(-1)
    return dequantize_at(f32(W).reshape(-1), idx).astype(np.float64).reshape(len(rows), K)


def oracle_cols(W, cols):
    """Dequantized columns `cols` of W [N, K] (float64), as [N, len(cols)]."""
    N, K = W.shape
    idx = (np.arange(N)[:, None] * K + np.asarray(cols)[None, :]).reshape(-1)
    return dequantize_at(f32(W).reshape(-1), idx).astype(np.float64).reshape(N, len(cols))


def sample(n, k, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=min(k, n), replace=False))


def check_codec_groups(W, Wp, seed, n_groups=48):
    """Packed codes and constants of sampled 256-block groups, bit for bit."""
    flat = f32(W).reshape(-1)
    n = flat.size
    groups = -(-n // 16384)
    pick = np.unique(np.concatenate([[0, groups - 1], sample(groups, n_groups, seed)]))
    codes, aq, sc = u8(Wp.codes), u8(Wp.absmax_q), Wp.absmax_scale.cpu().numpy()
    for g in pick:
        lo, hi = g * 16384, min(n, (g + 1) * 16384)
        oc, oq, osc = quantize_nf4(flat[lo:hi])
        np.testing.assert_array_equal(codes[lo // 2:(hi + 1) // 2], oc, err_msg=f"codes group {g}")
        np.testing.assert_array_equal(aq[lo // 64:-(-hi // 64)], oq, err_msg=f"absmax_q group {g}")
        np.testing.assert_array_equal(sc[g:g + 1], osc, err_msg=f"absmax_scale group {g}")


def run_linear(case, backward=True):
    Wp = q.qlora_quantize_nf4(case.W.to(DEV))
    X, A, B = (t.to(DEV) for t in (case.X, case.A, case.B))
    ws = q.new_workspace(case.M, case.K, case.N, case.r, DEV)
    Y, T = q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws)
    out = dict(Wp=Wp, Y=Y, T=T)
    if backward:
        dY = case.dY.to(DEV)
        dX, dA, dB = q.qlora_linear_bwd(dY, X, T, Wp, A, B, case.scale, workspace=ws)
        out.update(dX=dX, dA=dA, dB=dB)
    assert q.qlora_check_status(ws) == 0
    return out


def check_linear_sampled(case, g, seed, backward=True, n_rows=64, n_cols=64):
    X, A, B = f64(case.X), f64(case.A), f64(case.B)
    s = case.scale
    rows = sample(case.M, n_rows, seed)
    cols = sample(case.N, n_cols, seed + 1)
    Wr = oracle_rows(case.W, cols)                       # [n_cols, K]
    Yref = X[rows] @ Wr.T + (s * (X[rows] @ A)) @ B[:, cols]
    assert_close_rms(f64(g["Y"])[np.ix_(rows, cols)], Yref, "Y sampled")
    assert_close_rms(f64(g["T"]), s * (X @ A), "T")
    if not backward:
        return
    dY = f64(case.dY)
    kcols = sample(case.K, n_cols, seed + 2)
    Wc = oracle_cols(case.W, kcols)                      # [N, n_cols]
    U = s * (dY @ B.T)
    dXref = dY[rows] @ Wc + U[rows] @ A[kcols].T
    assert_close_rms(f64(g["dX"])[np.ix_(rows, kcols)], dXref, "dX sampled")
    assert_close_rms(f64(g["dA"]), X.T @ U, "dA")
    assert_close_rms(f64(g["dB"]), s * (X @ A).T @ dY, "dB")


# ------------------------------------------------------------- LLaMA-7B MLP trio
@pytest.mark.parametrize("name,K,N", [("gate_up", 4096, 11008), ("down", 11008, 4096)])
def test_mlp_trio_linear_shapes(name, K, N):
    """Each linear of the trio on its own (8192 tokens, r = 64, scale 0.25)."""
    case = synthetic.linear_case(8192, K, N, 64, 0.25, seed=2 if name == "gate_up" else 22)
    g = run_linear(case)
    check_codec_groups(case.W, g["Wp"], seed=5)
    check_linear_sampled(case, g, seed=7)


def test_mlp_trio_chain():
    """Y = down(silu(gate(X)) * up(X)) and its input gradient, on sampled rows.

    The SiLU gate is glue between the three LoRA linears (the library's
    elementwise kernels, float32 arithmetic, bf16 outputs); every linear runs
    through the library."""
    M, D, F, r = 8192, 4096, 11008, 64
    t = synthetic.mlp_trio(M, D, F, r, 0.25)
    s = t.scale
    Wg, Wu, Wd, X, dY = t.Wg, t.Wu, t.Wd, t.X, t.dY
    Ag, Au, Ad, Bg, Bu, Bd = t.Ag, t.Au, t.Ad, t.Bg, t.Bu, t.Bd

    d = lambda t: t.to(DEV)  # noqa: E731
    Pg, Pu, Pd = (q.qlora_quantize_nf4(d(w)) for w in (Wg, Wu, Wd))
    G, Tg = q.qlora_linear_fwd(d(X), Pg, d(Ag), d(Bg), s)
    Up, Tu = q.qlora_linear_fwd(d(X), Pu, d(Au), d(Bu), s)
    H = q.qlora_silu_gate_fwd(G, Up)
    Y, Td = q.qlora_linear_fwd(H, Pd, d(Ad), d(Bd), s)
    dH, _, _ = q.qlora_linear_bwd(d(dY), H, Td, Pd, d(Ad), d(Bd), s)
    dG, dU = q.qlora_silu_gate_bwd(G, Up, dH)
    dXg, _, _ = q.qlora_linear_bwd(dG, d(X), Tg, Pg, d(Ag), d(Bg), s)
    dXu, _, _ = q.qlora_linear_bwd(dU, d(X), Tu, Pu, d(Au), d(Bu), s)
    dX = dXg.float() + dXu.float()
    assert q.qlora_check_status(None) == 0

    rows = sample(M, 32, 11)
    Xr = f64(X)[rows]
    Wg_r = oracle_rows(Wg, np.arange(F))
    Wu_r = oracle_rows(Wu, np.arange(F))
    Wd_r = oracle_rows(Wd, np.arange(D))
    A_, B_ = {k: f64(v) for k, v in dict(g=Ag, u=Au, d=Ad).items()}, {k: f64(v) for k, v in dict(g=Bg, u=Bu, d=Bd).items()}
    # Each linear's output is bf16 by the layer contract, so the reference
    # chain rounds its own intermediates (G, Up, H, dH, dG, dUp) to bf16 the
    # same way; the gate arithmetic itself is float64.
    bf = lambda a: synthetic.to_bf16(a).double().numpy()  # noqa: E731
    Gr = bf(Xr @ Wg_r.T + s * (Xr @ A_["g"]) @ B_["g"])
    Ur = bf(Xr @ Wu_r.T + s * (Xr @ A_["u"]) @ B_["u"])
    sig = 1.0 / (1.0 + np.exp(-Gr))
    Hr = bf(Gr * sig * Ur)
    Yr = Hr @ Wd_r.T + s * (Hr @ A_["d"]) @ B_["d"]
    assert_close_rms(f64(Y)[rows], Yr, "trio Y rows")
    dYr = f64(dY)[rows]
    dHr = bf(dYr @ Wd_r + s * (dYr @ B_["d"].T) @ A_["d"].T)
    dGr = bf(dHr * Ur * sig * (1 + Gr * (1 - sig)))
    dUr = bf(dHr * Gr * sig)
    dXr = (dGr @ Wg_r + s * (dGr @ B_["g"].T) @ A_["g"].T) + (dUr @ Wu_r + s * (dUr @ B_["u"].T) @ A_["u"].T)
    assert_close_rms(dX[rows].double().cpu().numpy(), dXr, "trio dX rows")


# ------------------------------------------------------- LLaMA-65B-shaped linears
@pytest.mark.parametrize("name,K,N", [("qkvo", 8192, 8192), ("gate_up", 8192, 22016), ("down", 22016, 8192)])
def test_llama65b_linears(name, K, N):
    """4096 tokens, r = 64, scale 0.25 (seed 3 family)."""
    case = synthetic.linear_case(4096, K, N, 64, 0.25, seed=3 + K + N)
    g = run_linear(case)
    check_codec_groups(case.W, g["Wp"], seed=K)
    check_linear_sampled(case, g, seed=N)


def test_llama65b_quantize_all_seven_weights():
    """The one-shot quantization of the seven block weights, sampled groups."""
    shapes = [(8192, 8192)] * 4 + [(22016, 8192)] * 2 + [(8192, 22016)]
    for i, (n, k) in enumerate(shapes):
        W = synthetic.weight_only(n, k, seed=300 + i)
        Wp = q.qlora_quantize_nf4(W.to(DEV))
        check_codec_groups(W, Wp, seed=i, n_groups=16)


# --------------------------------------------------------------- small-M sweep
@pytest.mark.parametrize("N", [8192, 22016])
@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_small_m_forward(M, N):
    """Forward only, W [N x 8192], M tokens (seed 4)."""
    case = synthetic.small_m_case(M, N)
    g = run_linear(case, backward=False)
    check_linear_sampled(case, g, seed=M + N, backward=False, n_rows=M, n_cols=256)
