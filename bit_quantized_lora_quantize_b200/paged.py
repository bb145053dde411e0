"""Paged AdamW for the LoRA adapters (binding over libqlora.so).

"3. Paged Optimizers" ("QLoRA: Fine-Tuning 65-Billion Parameter Models on a
Single Consumer GPU") and "AI Glossary: QLoRA", second paragraph: only the
LoRA matrices are trained, and their optimizer states live in NVIDIA unified
memory, so they can move between GPU and CPU memory during memory spikes.

``PagedAdamW`` keeps, for a list of adapter shapes, one flat float32 master
copy of the parameters and the two AdamW moments in unified memory (torch
tensors allocated by the library's ``qlora_paged_malloc`` through a PyTorch
memory pool), and one flat bf16 buffer in ordinary device memory whose views
are the adapters the linear calls read.  The flat order matches
``dp.GradBucket``: (A [K, r], B [r, N]) per linear, so one library call
updates every adapter from one gradient bucket.  ``evict()`` moves the states
to host memory (before a spike), ``prefetch()`` brings them back (before the
step); a step on evicted states still runs, paging them in on demand.
"""

from __future__ import annotations

import ctypes

import torch

from . import qlora as q

_POOLS = {}


def paged_pool(device) -> "torch.cuda.MemPool":
    """A PyTorch memory pool whose blocks come from qlora_paged_malloc
    (unified memory), one per device."""
    dev = torch.device(device).index or 0
    if dev not in _POOLS:
        q.lib()
        from torch.cuda.memory import CUDAPluggableAllocator
        alloc = CUDAPluggableAllocator(q.LIB_PATH, "qlora_paged_malloc", "qlora_paged_free")
        _POOLS[dev] = (alloc, torch.cuda.MemPool(alloc.allocator()))
    return _POOLS[dev][1]


def paged_empty(n: int, dtype, device) -> torch.Tensor:
    with torch.cuda.use_mem_pool(paged_pool(device), device=device):
        return torch.empty(n, dtype=dtype, device=device)


def location(t: torch.Tensor) -> int:
    """Where the tensor's unified memory was last prefetched: a device index,
    or -1 for host memory."""
    loc = ctypes.c_int32(0)
    q._check("qlora_paged_location", q.lib().qlora_paged_location(t.data_ptr(), t.numel() * t.element_size(),
                                                                   ctypes.byref(loc)))
    return int(loc.value)


class PagedAdamW:
    """AdamW over the flattened adapters of several LoRA linears."""

    def __init__(self, shapes, device, lr=2e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0):
        """shapes: (K, N, r) per linear, in GradBucket order."""
        self.shapes = list(shapes)
        self.n = sum(K * r + r * N for K, N, r in self.shapes)
        self.device = torch.device(device)
        self.lr, self.betas, self.eps, self.wd = float(lr), tuple(betas), float(eps), float(weight_decay)
        self.master = paged_empty(self.n, torch.float32, self.device)
        self.m = paged_empty(self.n, torch.float32, self.device)
        self.v = paged_empty(self.n, torch.float32, self.device)
        self.m.zero_()
        self.v.zero_()
        self.params = torch.empty(self.n, dtype=torch.bfloat16, device=self.device)
        self.views = []
        off = 0
        for K, N, r in self.shapes:
            A = self.params[off:off + K * r].view(K, r)
            off += K * r
            B = self.params[off:off + r * N].view(r, N)
            off += r * N
            self.views.append((A, B))
        self.t = 0

    def load(self, adapters) -> None:
        """Initial adapters: a list of (A, B) bf16 tensors, one per linear."""
        for (A, B), (a, b) in zip(self.views, adapters):
            A.copy_(a)
            B.copy_(b)
        self.master.copy_(self.params.float())

    def step(self, grads: torch.Tensor) -> None:
        """One AdamW step from the flat float32 gradient bucket."""
        if grads.numel() != self.n or grads.dtype != torch.float32 or not grads.is_cuda:
            raise ValueError("grads must be the flat float32 CUDA gradient bucket of these shapes")
        self.t += 1
        b1, b2 = self.betas
        q._check("qlora_adamw_step", q.lib().qlora_adamw_step(
            self.master.data_ptr(), self.params.data_ptr(), grads.data_ptr(), self.m.data_ptr(), self.v.data_ptr(),
            self.n, self.t, self.lr, b1, b2, self.eps, self.wd, torch.cuda.current_stream().cuda_stream))

    def _move(self, to_device: int) -> None:
        st = torch.cuda.current_stream().cuda_stream
        for t in (self.master, self.m, self.v):
            q._check("qlora_paged_prefetch", q.lib().qlora_paged_prefetch(t.data_ptr(), t.numel() * 4, to_device, st))

    def evict(self) -> None:
        """Move the optimizer states to host memory (asynchronous, on the
        current stream)."""
        self._move(0)

    def prefetch(self) -> None:
        """Bring the optimizer states back to the GPU (asynchronous)."""
        self._move(1)

    @property
    def state_bytes(self) -> int:
        return 3 * self.n * 4


__all__ = ["PagedAdamW", "paged_pool", "paged_empty", "location"]
