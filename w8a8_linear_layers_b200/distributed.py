"""Data-parallel plumbing for the W8A8 path (torch.distributed).

Each rank is a replica of the linear layer with its own batch of tokens.  The
only exchange the path needs is the calibration statistic: the per-input-
channel activation absmax (SmoothQuant's max|X_j|, "SmoothQuant大模型量化技术
深度解析", section 1) must be the max over the whole global batch, so every
replica derives the same smoothing factor and the same quantized weight.  MAX
is exact and order-free, so the result is bit-identical to a single device
seeing all tokens.  Everything after calibration is rank-local.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world_size(group=None) -> int:
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def allreduce_calibration(absmax: torch.Tensor, group=None) -> None:
    """In place: absmax <- max over ranks (no-op on one rank)."""
    if world_size(group) > 1:
        dist.all_reduce(absmax, op=dist.ReduceOp.MAX, group=group)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest of a per-rank scalar (e.g. a device time), on every rank."""
    if world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
