"""Data-parallel exchange for the QLoRA layer.

With the frozen 4-bit base replicated on every rank and the tokens split across
ranks, the only quantities that cross ranks are the adapter gradients dA (r x k)
and dB (d x r).  They live as views into one flat fp32 bucket so a step needs a
single all-reduce (NCCL over NVLink on GPUs; gloo in the CPU tests).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch
import torch.distributed as dist


class GradBucket:
    """One contiguous fp32 buffer carved into gradient views."""

    def __init__(self, shapes: Sequence[Tuple[int, ...]], device):
        sizes = [int(torch.Size(s).numel()) for s in shapes]
        # keep every view 16-byte aligned (the kernels write with 16-byte stores)
        offsets, off = [], 0
        for n in sizes:
            offsets.append(off)
            off += (n + 3) // 4 * 4
        self.flat = torch.zeros(max(off, 4), dtype=torch.float32, device=device)
        self.views: List[torch.Tensor] = [self.flat[o:o + n].view(s) for o, n, s in zip(offsets, sizes, shapes)]

    def allreduce(self, group=None) -> None:
        """Sum the bucket over all ranks of `group`, in place."""
        if dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (timings are reported as the max)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
