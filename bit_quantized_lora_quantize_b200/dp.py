"""Data-parallel plumbing for the frozen-NF4 LoRA linear layer.

Each rank holds the packed frozen weight and the adapter and processes its
own tokens; the forward and the input gradient need no communication.  The
one exchange step is the sum of the adapter gradients over ranks ("AI
Glossary: QLoRA", second paragraph: only the LoRA matrices get weight
gradients), done as a single all-reduce of one flat float32 buffer.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def shard_rows(M: int, rank: int, world: int) -> slice:
    """Contiguous share of M token rows for `rank` (sizes differ by at most 1)."""
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


class AdapterGradReducer:
    """Sums dA [K, r] and dB [r, N] over the process group in one collective."""

    def __init__(self, K: int, N: int, r: int, device, group=None):
        self.K, self.N, self.r = K, N, r
        self.group = group
        self.buf = torch.empty(K * r + r * N, dtype=torch.float32, device=device)

    def __call__(self, dA: torch.Tensor, dB: torch.Tensor) -> None:
        n_a = self.K * self.r
        self.buf[:n_a].copy_(dA.reshape(-1))
        self.buf[n_a:].copy_(dB.reshape(-1))
        dist.all_reduce(self.buf, op=dist.ReduceOp.SUM, group=self.group)
        dA.copy_(self.buf[:n_a].view_as(dA))
        dB.copy_(self.buf[n_a:].view_as(dB))


__all__ = ["shard_rows", "AdapterGradReducer"]
