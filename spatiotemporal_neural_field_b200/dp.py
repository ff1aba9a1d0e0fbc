"""Host-side data-parallel plumbing (one process per GPU, torch.distributed).

The decoder's positions are independent, so N ranks decode N independent
position sets with no exchange on the forward path (weak scaling).  A
data-parallel training step has exactly one exchange: the sum of the table
and weight gradients before the (replicated) Adam update.  Timings are taken
as the maximum over ranks.  Works with any backend (NCCL on GPUs, gloo on
CPU for tests).
"""
from __future__ import annotations

from typing import Iterable

import torch
import torch.distributed as dist


def world() -> int:
    return dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1


def rank() -> int:
    return dist.get_rank() if dist.is_available() and dist.is_initialized() else 0


def rank_frame(base_frame: int, r: int, n_frames: int) -> int:
    """The frame a rank decodes in a weak-scaling run: consecutive frames."""
    return (base_frame + r) % n_frames


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if world() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_gradients(tensors: Iterable[torch.Tensor]) -> None:
    """Sum gradient tensors over ranks in place (before a replicated Adam)."""
    if world() == 1:
        return
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
