"""Data-parallel plumbing for the adapted linear layers (host side).

QLoRA trains only the adapters ("QLoRA", ozercemkelahmet.com, How it works,
Step 6), so the data-parallel step exchanges exactly one thing: the fp32 adapter
gradients dA and dB, which are sums over tokens and therefore add across ranks.
The frozen NF4 weight is identical on every rank (quantization is
deterministic), so it is never communicated.  Everything here is torch
plumbing: one flat fp32 bucket whose views are handed to the library as the
dA / dB outputs, and one all-reduce per step.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch


def shard_tokens(m_global: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous token range [lo, hi) of `rank` out of `world` (sizes differ by <= 1)."""
    base, extra = divmod(m_global, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


class GradBucket:
    """One flat fp32 buffer holding dA [K, r] and dB [r, N] of several layers."""

    def __init__(self, shapes: Sequence[Tuple[int, int, int]], device, dtype=torch.float32):
        """shapes: (N, K, r) per layer."""
        total = sum(K * r + r * N for (N, K, r) in shapes)
        self.flat = torch.zeros(total, dtype=dtype, device=device)
        self.views: List[Tuple[torch.Tensor, torch.Tensor]] = []
        off = 0
        for (N, K, r) in shapes:
            dA = self.flat[off:off + K * r].view(K, r)
            off += K * r
            dB = self.flat[off:off + r * N].view(r, N)
            off += r * N
            self.views.append((dA, dB))

    def allreduce_(self, group=None) -> None:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
