"""Data-parallel plumbing for the W8A8 path (torch.distributed).

Each rank is a replica of the linear layer with its own batch of tokens.  The
only exchange the path needs is the calibration statistic: the per-input-
channel activation absmax (SmoothQuant's max|X_j|, "SmoothQuant大模型量化技术
深度解析", section 1) must be the max over the whole global batch, so every
replica derives the same smoothing factor and the same quantized weight.  MAX
is exact and order-free, so the result is bit-identical to a single device
seeing all tokens.  Everything after calibration is rank-local.

row_parallel_linear is the other sharding the path admits: the input
channels K split across ranks (RowParallelLinear), with a MAX exchange of
the per-token scales and an exact int32 SUM of the partial products.
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


# ------------------------------------------------------------ K-sharded linear
class KernelOps:
    """The library kernels the K-sharded linear runs on each rank."""

    def __init__(self, lib_module=None):
        if lib_module is None:
            import w8a8_linear_layers_b200 as lib_module
        self.w = lib_module

    def per_token_scales(self, x: torch.Tensor, inv_s: torch.Tensor | None) -> torch.Tensor:
        q = torch.empty(x.shape, device=x.device, dtype=torch.int8)
        sx = torch.empty(x.shape[0], device=x.device, dtype=torch.float32)
        self.w.quant_act_per_token(x, inv_s, q, sx)
        return sx

    def quant_given(self, x, inv_s, sx) -> torch.Tensor:
        q = torch.empty(x.shape, device=x.device, dtype=torch.int8)
        self.w.quant_act_given_scale(x, inv_s, sx, q)
        return q

    def gemm_acc(self, qx, qw, sx, sw) -> torch.Tensor:
        M, N = qx.shape[0], qw.shape[0]
        acc = torch.empty(M, N, device=qx.device, dtype=torch.int32)
        scratch_y = torch.empty(M, N, device=qx.device, dtype=torch.float32)  # dequant of a partial: unused
        self.w.w8a8_gemm_dequant(qx, sx, qw, sw, scratch_y, acc_out=acc)
        return acc

    def dequant(self, acc, sx, sw, y) -> None:
        self.w.sq_dequant(acc, sx, sw, y)


def row_parallel_linear(x_shard: torch.Tensor, inv_s_shard: torch.Tensor | None, qw_shard: torch.Tensor,
                        sw: torch.Tensor, y: torch.Tensor, group=None, ops=None) -> torch.Tensor:
    """y = the W8A8 linear of a layer whose input channels K are split across
    ranks (RowParallelLinear): rank r holds x[:, K_r], inv_s[K_r] and the
    codes qw[:, K_r]; sw (all N) and y (all of it) are replicated.

    1. local per-token scales fl(max_r / 127); all-reduce MAX -> the
       unsharded scales (x -> fl(x / 127) is monotonic);
    2. codes of the local slice at those scales;
    3. local int32 product; all-reduce SUM (exact);
    4. dequant of the sum.
    Every rank ends with the unsharded result, bit for bit."""
    ops = ops or KernelOps()
    sx = ops.per_token_scales(x_shard, inv_s_shard)
    if world_size(group) > 1:
        dist.all_reduce(sx, op=dist.ReduceOp.MAX, group=group)
    qx = ops.quant_given(x_shard, inv_s_shard, sx)
    acc = ops.gemm_acc(qx, qw_shard, sx, sw)
    if world_size(group) > 1:
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    ops.dequant(acc, sx, sw, y)
    return y
