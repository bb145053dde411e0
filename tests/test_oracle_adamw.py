"""Pins for the oracle's AdamW step ("3. Paged Optimizers": the optimizer
states of the LoRA parameters; the step itself is the textbook AdamW, see
oracle/adamw_ref.py).

* First step from zero states: mh = g and vh = g^2, so each parameter moves
  by lr * (g / (|g| + eps) + wd * p) -- about lr in the gradient's sign.
* A constant gradient keeps mh = g and vh = g^2 at every step, so with
  wd = 0 the parameters move by the same amount each step (a closed form).
* torch.optim.AdamW (float64, CPU) -- an independent library implementation.
* Zero gradient with wd = 0 leaves the parameters unchanged.
"""

import numpy as np
import torch

from oracle import adamw_run, adamw_step


def test_first_step_closed_form():
    rng = np.random.default_rng(0)
    p = rng.standard_normal(1000) * 0.01
    g = rng.standard_normal(1000)
    lr, eps, wd = 1e-3, 1e-8, 0.01
    p1, m1, v1 = adamw_step(p, g, np.zeros(1000), np.zeros(1000), 1, lr, eps=eps, wd=wd)
    np.testing.assert_allclose(p1, p - lr * (g / (np.abs(g) + eps) + wd * p), rtol=1e-13, atol=1e-18)
    np.testing.assert_allclose(m1, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v1, 0.001 * g * g, rtol=1e-13)


def test_constant_gradient_moves_linearly():
    g = np.array([0.5, -2.0, 1e-3, 7.0])
    lr, eps = 2e-4, 1e-8
    for t in (1, 2, 5, 17):
        p, _, _ = adamw_run(np.zeros(4), [g] * t, lr, eps=eps)
        np.testing.assert_allclose(p, -t * lr * g / (np.abs(g) + eps), rtol=1e-12)


def test_zero_gradient_without_decay_is_a_fixed_point():
    p0 = np.linspace(-1, 1, 17)
    p, m, v = adamw_run(p0, [np.zeros(17)] * 3, 1e-2)
    np.testing.assert_array_equal(p, p0)
    assert not m.any() and not v.any()


def test_matches_torch_adamw_in_float64():
    rng = np.random.default_rng(1)
    p0 = rng.standard_normal((64, 48)) * 0.02
    grads = [rng.standard_normal((64, 48)) for _ in range(6)]
    lr, b1, b2, eps, wd = 3e-4, 0.9, 0.95, 1e-6, 0.1
    p_ref, _, _ = adamw_run(p0, grads, lr, b1, b2, eps, wd)
    t = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([t], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    for g in grads:
        t.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
    np.testing.assert_allclose(p_ref, t.detach().numpy(), rtol=1e-12, atol=1e-15)
