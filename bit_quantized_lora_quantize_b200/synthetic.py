"""Seeded synthetic inputs for the frozen-NF4 LoRA linear layer.

This module only draws random numbers and stores them as bfloat16; it holds
none of the method's arithmetic.  Both the CUDA path (tests, bench) and the
CPU oracle consume exactly the tensors it returns.

Recipe: numpy PCG64 seeded by ``SeedSequence(seed)``, one spawned child per
tensor in a fixed order (W, outlier mask, X, A, B, dY, extra inputs); draws
in float32, stored as bfloat16 by round-to-nearest-even (torch's conversion).
The workloads follow the layer shapes of the LLaMA family used in the QLoRA
experiments: weights ~ N(0, 0.02^2), activations and upstream gradients
~ N(0, 1), LoRA factors ~ N(0, 0.01^2) (or U(-1/16, 1/16) for the small
parity case), optionally a fraction of weight entries multiplied by 10 to
mimic outlier features.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

_STREAMS = ("W", "outliers", "X", "A", "B", "dY", "extra0", "extra1", "extra2", "extra3")


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32/float64 numpy array -> CPU bfloat16 tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


class Streams:
    """Independent PCG64 generators, one per named tensor, from one seed."""

    def __init__(self, seed: int):
        kids = np.random.SeedSequence(seed).spawn(len(_STREAMS))
        self._rng = {name: np.random.Generator(np.random.PCG64(k)) for name, k in zip(_STREAMS, kids)}

    def __getitem__(self, name: str) -> np.random.Generator:
        return self._rng[name]


def normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)


def uniform(rng: np.random.Generator, shape, half_width: float) -> np.ndarray:
    u = rng.random(shape, dtype=np.float32)
    return (u * np.float32(2.0) - np.float32(1.0)) * np.float32(half_width)


@dataclass
class LinearCase:
    """One LoRA linear layer's inputs (CPU bfloat16 tensors) and its scale."""

    W: torch.Tensor    # [N, K]
    X: torch.Tensor    # [M, K]
    A: torch.Tensor    # [K, r]
    B: torch.Tensor    # [r, N]
    dY: torch.Tensor   # [M, N]
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def M(self) -> int:
        return self.X.shape[0]

    @property
    def K(self) -> int:
        return self.X.shape[1]

    @property
    def N(self) -> int:
        return self.W.shape[0]

    @property
    def r(self) -> int:
        return self.A.shape[1]


def linear_case(M: int, K: int, N: int, r: int, scale: float, seed: int, *,
                w_std: float = 0.02, outlier_frac: float = 0.0,
                a_dist: str = "normal", a_param: float = 0.01, b_std: float = 0.01,
                with_dy: bool = True) -> LinearCase:
    """Draw one layer's inputs.  ``a_dist`` is "normal" (std a_param) or
    "uniform" (half-width a_param)."""
    st = Streams(seed)
    w = normal(st["W"], (N, K), w_std)
    n_out = int(round(outlier_frac * N * K))
    if n_out:
        idx = st["outliers"].choice(N * K, size=n_out, replace=False)
        w.reshape(-1)[idx] *= np.float32(10.0)
    x = normal(st["X"], (M, K), 1.0)
    if a_dist == "uniform":
        a = uniform(st["A"], (K, r), a_param)
    else:
        a = normal(st["A"], (K, r), a_param)
    b = normal(st["B"], (r, N), b_std)
    dy = normal(st["dY"], (M, N), 1.0) if with_dy else np.zeros((0, N), np.float32)
    return LinearCase(W=to_bf16(w), X=to_bf16(x), A=to_bf16(a), B=to_bf16(b), dY=to_bf16(dy),
                      scale=float(scale), meta=dict(seed=seed, outlier_frac=outlier_frac))


def weight_only(rows: int, cols: int, seed: int, std: float = 0.02) -> torch.Tensor:
    """A bf16 weight ~ N(0, std^2) from the 'W' stream of ``seed``."""
    return to_bf16(normal(Streams(seed)["W"], (rows, cols), std))


# Named workloads ----------------------------------------------------------

def tiny_case() -> LinearCase:
    """Single QLoRA linear, 256 x 256, 16 tokens, r = 8, scale 2 (seed 0)."""
    return linear_case(16, 256, 256, 8, 2.0, 0, a_dist="uniform", a_param=1.0 / 16.0)


def attn_proj_case() -> LinearCase:
    """LLaMA-7B attention projection: W 4096 x 4096 with 0.1% of entries x10,
    4096 tokens, r = 64, scale 0.25 (seed 1)."""
    return linear_case(4096, 4096, 4096, 64, 0.25, 1, outlier_frac=0.001)


def small_m_case(M: int, N: int, K: int = 8192, seed: int = 4) -> LinearCase:
    """Small-M forward: W N x K, M tokens, r = 64, scale 0.25 (no dY)."""
    return linear_case(M, K, N, 64, 0.25, seed, with_dy=False)


# The seven linears of a LLaMA-65B-shaped block: (name, out N, in K).
LLAMA65B_LINEARS = (("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
                    ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016))


def llama65b_block(M: int = 4096, r: int = 64, scale: float = 0.25) -> list:
    """LLaMA-65B-shaped block linears, M tokens (seed family 3).

    Weight i is the 'W' stream of seed 300 + i (the same weights the one-shot
    quantization test uses); the six linears with in-dim 8192 share one input
    X (the 'X' stream of seed 3); the down projection takes its own
    M x 22016 input (the 'extra0' stream of seed 3).  Adapter i and its dY
    come from the A, B and dY streams of seed 310 + i.  Returns a list of
    (name, LinearCase)."""
    st = Streams(3)
    X = to_bf16(normal(st["X"], (M, 8192), 1.0))
    Xd = to_bf16(normal(st["extra0"], (M, 22016), 1.0))
    out = []
    for i, (name, N, K) in enumerate(LLAMA65B_LINEARS):
        w = weight_only(N, K, seed=300 + i)
        sa = Streams(310 + i)
        a = to_bf16(normal(sa["A"], (K, r), 0.01))
        b = to_bf16(normal(sa["B"], (r, N), 0.01))
        dy = to_bf16(normal(sa["dY"], (M, N), 1.0))
        out.append((name, LinearCase(W=w, X=X if K == 8192 else Xd, A=a, B=b, dY=dy, scale=float(scale),
                                     meta=dict(seed=300 + i))))
    return out


@dataclass
class MlpTrio:
    """LLaMA-7B MLP: gate/up [F x D], down [D x F], X [M x D], dY [M x D]."""

    Wg: torch.Tensor
    Wu: torch.Tensor
    Wd: torch.Tensor
    X: torch.Tensor
    Ag: torch.Tensor
    Au: torch.Tensor
    Ad: torch.Tensor
    Bg: torch.Tensor
    Bu: torch.Tensor
    Bd: torch.Tensor
    dY: torch.Tensor
    scale: float


def mlp_trio(M: int = 8192, D: int = 4096, F: int = 11008, r: int = 64, scale: float = 0.25) -> MlpTrio:
    """LLaMA-7B MLP trio inputs (seed 2), drawn in a fixed stream order."""
    st = Streams(2)
    Wg = to_bf16(normal(st["W"], (F, D), 0.02))
    Wu = to_bf16(normal(st["outliers"], (F, D), 0.02))
    Wd = to_bf16(normal(st["extra0"], (D, F), 0.02))
    X = to_bf16(normal(st["X"], (M, D), 1.0))
    Ag, Au = (to_bf16(normal(st["A"], (D, r), 0.01)) for _ in range(2))
    Ad = to_bf16(normal(st["A"], (F, r), 0.01))
    Bg, Bu = (to_bf16(normal(st["B"], (r, F), 0.01)) for _ in range(2))
    Bd = to_bf16(normal(st["B"], (r, D), 0.01))
    dY = to_bf16(normal(st["dY"], (M, D), 1.0))
    return MlpTrio(Wg, Wu, Wd, X, Ag, Au, Ad, Bg, Bu, Bd, dY, float(scale))


__all__ = ["to_bf16", "Streams", "LinearCase", "linear_case", "weight_only",
           "tiny_case", "attn_proj_case", "small_m_case", "LLAMA65B_LINEARS", "llama65b_block",
           "MlpTrio", "mlp_trio"]
