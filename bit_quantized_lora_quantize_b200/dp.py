"""Data-parallel plumbing for the frozen-NF4 LoRA linear layer.

Each rank holds the packed frozen weights and the adapters and processes its
own tokens; the forward and the input gradient need no communication.  The
one exchange step is the sum of the adapter gradients over ranks ("AI
Glossary: QLoRA", second paragraph: only the LoRA matrices get weight
gradients).  The gradients of every linear of a step live in one flat
float32 bucket: the backward writes dA and dB straight into views of it, and
one all-reduce per step sums the whole bucket in place (no pack or unpack
copies, one collective launch).
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def shard_rows(M: int, rank: int, world: int) -> slice:
    """Contiguous share of M token rows for `rank` (sizes differ by at most 1)."""
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


class GradBucket:
    """dA [K, r] and dB [r, N] of several linears as views of one flat
    float32 buffer, in the order the shapes are given."""

    def __init__(self, shapes, device):
        """shapes: iterable of (K, N, r), one per linear."""
        shapes = list(shapes)
        total = sum(K * r + r * N for K, N, r in shapes)
        self.flat = torch.zeros(total, dtype=torch.float32, device=device)
        self.views = []
        off = 0
        for K, N, r in shapes:
            dA = self.flat[off:off + K * r].view(K, r)
            off += K * r
            dB = self.flat[off:off + r * N].view(r, N)
            off += r * N
            self.views.append((dA, dB))

    def __getitem__(self, i):
        return self.views[i]

    def __len__(self):
        return len(self.views)

    @property
    def nbytes(self) -> int:
        return self.flat.numel() * 4

    def all_reduce(self, group=None) -> None:
        """Sum the bucket over the process group, in place."""
        dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)


__all__ = ["shard_rows", "GradBucket"]
