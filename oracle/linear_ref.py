"""Oracle for the frozen-NF4 linear layer with a LoRA adapter: forward and
backward, exact linear algebra in float64.

TEST INFRASTRUCTURE ONLY (see the package header).

Notation.  W' in bf16[N x K] is the dequantized frozen weight (out x in,
row-major, the layout a linear layer stores); X in bf16[M x K];
A in bf16[K x r]; B in bf16[r x N]; s is the float LoRA scale.

* "QLoRA: Fine-Tuning 65-Billion Parameter Models ...", section "LoRA:
  Prerequisite for Understanding QLoRA": the update of a d x k weight is the
  product of a d x r and an r x k matrix.  Read with A = [in x r] and
  B = [r x out], i.e. the stored W' is the transpose of the page's d x k.
* "AI Glossary: QLoRA", second paragraph: the 4-bit weights are turned back
  into BFloat16 for the calculation, and weight gradients are computed only
  for the LoRA matrices; "QLoRA's Working Process", step 5: gradients flow
  through the frozen 4-bit model to the adapters.
* The LoRA scale s is not defined on the pages (the "Optimization Tips" list
  gives alpha = 2 x rank as typical); it is an argument here.

Definitions (no intermediate rounding; inputs are the exact bf16 values):
    T  = s * X A                           (M x r)
    Y  = X W'^T + T B                      (M x N)
    given dY (M x N), for L = sum(Y * dY):
    dX = dY W' + s * (dY B^T) A^T          (M x K)
    dA = s * X^T (dY B^T)                  (K x r)
    dB = s * (X A)^T dY                    (r x N)
No gradient of W' exists: the base weight is frozen.
"""

from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def lora_linear_forward(X, Wdq, A, B, s: float):
    """Return ``(Y, T)`` in float64: Y = X W'^T + s (X A) B, T = s X A."""
    X, Wdq, A, B = _f64(X), _f64(Wdq), _f64(A), _f64(B)
    T = float(s) * (X @ A)
    Y = X @ Wdq.T + T @ B
    return Y, T


def lora_linear_backward(dY, X, Wdq, A, B, s: float):
    """Return ``(dX, dA, dB)`` in float64 for L = sum(Y * dY)."""
    dY, X, Wdq, A, B = _f64(dY), _f64(X), _f64(Wdq), _f64(A), _f64(B)
    s = float(s)
    U = s * (dY @ B.T)          # M x r
    dX = dY @ Wdq + U @ A.T
    dA = X.T @ U
    dB = s * (X @ A).T @ dY
    return dX, dA, dB


__all__ = ["lora_linear_forward", "lora_linear_backward"]
