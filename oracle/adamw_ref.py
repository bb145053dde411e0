"""Oracle for the optimizer step of the LoRA parameters (AdamW).

TEST INFRASTRUCTURE ONLY (see the package header).  numpy float64.

What the pages fix: "AI Glossary: QLoRA", second paragraph, and "3. Paged
Optimizers" in "QLoRA: Fine-Tuning 65-Billion Parameter Models ...": only the
LoRA matrices are trained, and their optimizer states live in NVIDIA unified
memory so that they can move between GPU and CPU memory during memory spikes
("paging").  The pages name no optimizer formula.  Reading: the optimizer is
AdamW (Adam with decoupled weight decay), the plain textbook step, with the
paging being where the states are stored, not what is computed:

    m_t = b1 m_{t-1} + (1 - b1) g
    v_t = b2 v_{t-1} + (1 - b2) g^2
    mh  = m_t / (1 - b1^t),   vh = v_t / (1 - b2^t)
    p_t = p_{t-1} - lr (mh / (sqrt(vh) + eps) + wd p_{t-1})

with t counted from 1 and m_0 = v_0 = 0.  The trained adapter is kept as a
float32 master copy; the bf16 adapter the linear layer reads is its
round-to-nearest-even bf16 value.
"""

from __future__ import annotations

import numpy as np


def adamw_step(p, g, m, v, t: int, lr: float, b1: float = 0.9, b2: float = 0.999, eps: float = 1e-8,
               wd: float = 0.0):
    """One AdamW step in float64.  Returns ``(p_new, m_new, v_new)``."""
    p, g, m, v = (np.asarray(a, dtype=np.float64) for a in (p, g, m, v))
    if t < 1:
        raise ValueError("step count starts at 1")
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    mh = m / (1.0 - b1 ** t)
    vh = v / (1.0 - b2 ** t)
    p = p - lr * (mh / (np.sqrt(vh) + eps) + wd * p)
    return p, m, v


def adamw_run(p0, grads, lr: float, b1: float = 0.9, b2: float = 0.999, eps: float = 1e-8, wd: float = 0.0):
    """Steps 1..len(grads) from p0 with zero states; returns the final
    ``(p, m, v)``."""
    p = np.asarray(p0, dtype=np.float64)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    for t, g in enumerate(grads, start=1):
        p, m, v = adamw_step(p, g, m, v, t, lr, b1, b2, eps, wd)
    return p, m, v


__all__ = ["adamw_step", "adamw_run"]
