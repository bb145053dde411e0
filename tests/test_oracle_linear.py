"""Pins for the oracle's LoRA linear forward and backward.

"AI Glossary: QLoRA", second paragraph: weight gradients exist only for the
LoRA matrices; "QLoRA's Working Process", step 5: gradients flow through the
frozen 4-bit weights into the adapters.  The backward is pinned by central
finite differences of L = sum(Y * dY) (which checks every term, sign and
transpose), by torch's float64 autograd (a library routine), and by the
special cases B = 0, A = 0 and s = 0.
"""

import numpy as np
import pytest
import torch

from oracle import lora_linear_forward, lora_linear_backward


def small(seed, M=5, K=12, N=7, r=3):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) * 0.1
    A = rng.standard_normal((K, r)) * 0.3
    B = rng.standard_normal((r, N)) * 0.3
    dY = rng.standard_normal((M, N))
    return X, W, A, B, dY


def loss(X, W, A, B, dY, s):
    Y, _ = lora_linear_forward(X, W, A, B, s)
    return float(np.sum(Y * dY))


@pytest.mark.parametrize("s", [2.0, 0.25, -1.5])
def test_backward_matches_central_differences(s):
    X, W, A, B, dY = small(1)
    dX, dA, dB = lora_linear_backward(dY, X, W, A, B, s)
    h = 1e-6
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(P)
        for idx in np.ndindex(P.shape):
            P[idx] += h
            lp = loss(X, W, A, B, dY, s)
            P[idx] -= 2 * h
            lm = loss(X, W, A, B, dY, s)
            P[idx] += h
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(G, num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_forward_backward_match_torch_autograd_fp64():
    X, W, A, B, dY = small(2, M=9, K=16, N=11, r=4)
    s = 0.75
    tX, tA, tB = (torch.tensor(v, requires_grad=True) for v in (X, A, B))
    tW = torch.tensor(W)
    Y = torch.nn.functional.linear(tX, tW) + s * (tX @ tA) @ tB
    Y.backward(torch.tensor(dY))
    oY, oT = lora_linear_forward(X, W, A, B, s)
    dX, dA, dB = lora_linear_backward(dY, X, W, A, B, s)
    np.testing.assert_allclose(oY, Y.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oT, s * X @ A, rtol=1e-12, atol=1e-12)
    for got, ref in ((dX, tX.grad), (dA, tA.grad), (dB, tB.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_special_cases():
    X, W, A, B, dY = small(3)
    # B = 0: no adapter gradient reaches A; Y is the frozen product alone.
    Z = np.zeros_like(B)
    Y, _ = lora_linear_forward(X, W, A, Z, 1.0)
    _, dA, _ = lora_linear_backward(dY, X, W, A, Z, 1.0)
    assert np.all(dA == 0.0)
    np.testing.assert_allclose(Y, torch.nn.functional.linear(torch.tensor(X), torch.tensor(W)).numpy(),
                               rtol=1e-13, atol=1e-13)
    # A = 0: T = 0 and dB = 0.
    Y, T = lora_linear_forward(X, W, np.zeros_like(A), B, 1.0)
    _, _, dB = lora_linear_backward(dY, X, W, np.zeros_like(A), B, 1.0)
    assert np.all(T == 0.0) and np.all(dB == 0.0)
    # s = 0: the dense layer, dX = dY W.
    Y, _ = lora_linear_forward(X, W, A, B, 0.0)
    dX, dA, dB = lora_linear_backward(dY, X, W, A, B, 0.0)
    np.testing.assert_allclose(Y, X @ W.T, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dX, dY @ W, rtol=1e-13, atol=1e-13)
    assert np.all(dA == 0.0) and np.all(dB == 0.0)
