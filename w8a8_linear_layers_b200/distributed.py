"""Data-parallel plumbing for the W8A8 path (torch.distributed).

Each rank is a replica of the linear layer with its own batch of tokens.  The
only exchange the path needs is the calibration statistic: the per-input-
channel activation absmax (SmoothQuant's max|X_j|, "SmoothQuant大模型量化技术
深度解析", section 1) must be the max over the whole global batch, so every
replica derives the same smoothing factor and the same quantized weight.  MAX
is exact and order-free, so the result is bit-identical to a single device
seeing all tokens.  Everything after calibration is rank-local.

row_parallel_linear is one of the two shardings of a single layer: the
input channels K split across ranks (RowParallelLinear), with a MAX exchange
of the per-token scales and an exact int32 SUM of the partial products.
column_parallel_linear is the other: the output channels N split across
ranks (ColumnParallelLinear, "PaddleNLP GPT 量化感知训练（QAT）实战指南"
section 5.2, tensor-parallel degree 8), X replicated, no exchange but an
optional all-gather of Y.  ssz_quant_weight_sharded splits the SSZ search by
output channel the same way: the channels are independent (each stops on its
own test), so each rank searches its block and an all-gather gives every
rank the whole quantized weight, bit-identical to one device doing it all.
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

    def ssz(self, w_rows, s, bits, max_iters, q_out, scale_out, iters_out) -> None:
        self.w.ssz_quant_weight(w_rows, s, bits, max_iters, q_out, scale_out, iters_out=iters_out)

    def quant_act(self, x, inv_s, qx, sx) -> None:
        self.w.quant_act_per_token(x, inv_s, qx, sx)

    def gemm(self, qx, sx, qw, sw, y) -> None:
        self.w.w8a8_gemm_dequant(qx, sx, qw, sw, y)


def rank(group=None) -> int:
    return dist.get_rank(group) if dist.is_available() and dist.is_initialized() else 0


def shard_rows(n: int, world: int, r: int) -> tuple[int, int]:
    """Rank r's contiguous block [a, b) of n rows split over `world` ranks
    (sizes differ by at most one, the larger blocks first)."""
    base, rem = divmod(n, world)
    a = r * base + min(r, rem)
    return a, a + base + (1 if r < rem else 0)


def _gather_rows(local: torch.Tensor, out: torch.Tensor, n: int, group=None) -> None:
    """out[a_r:b_r] <- rank r's local[:b_r - a_r] for every rank (the blocks of
    shard_rows; local is padded to the largest block)."""
    G = world_size(group)
    # moved as bytes (a bit copy, and every backend gathers uint8), one row of
    # bytes per row of the tensor
    if local.dim() == 1:
        local, out = local.unsqueeze(1), out.unsqueeze(1)
    local, out = local.contiguous().view(torch.uint8), out.view(torch.uint8)
    parts = [torch.empty_like(local) for _ in range(G)]
    dist.all_gather(parts, local, group=group)
    for r, part in enumerate(parts):
        a, b = shard_rows(n, G, r)
        out[a:b].copy_(part[: b - a])


def ssz_quant_weight_sharded(w: torch.Tensor, s: torch.Tensor | None, bits: int, max_iters: int, q_out: torch.Tensor,
                             scale_out: torch.Tensor, iters_out: torch.Tensor | None = None, group=None,
                             ops=None) -> None:
    """ssz_quant_weight of the whole [N, K] weight w (present on every rank),
    with the output channels split across ranks: rank r searches the block
    shard_rows(N, G, r), then the codes, scales and rounds of all blocks are
    all-gathered into q_out [N, K], scale_out [N] and iters_out [N] on every
    rank.  Channels are independent, so the result is the unsharded one bit
    for bit; each rank does 1/G of the search."""
    ops = ops or KernelOps()
    G, N = world_size(group), w.shape[0]
    if G == 1:
        its = iters_out if iters_out is not None else torch.empty(N, dtype=torch.int32, device=w.device)
        ops.ssz(w, s, bits, max_iters, q_out, scale_out, its)
        return
    a, b = shard_rows(N, G, rank(group))
    rmax = -(-N // G)
    q_loc = torch.zeros(rmax, w.shape[1], dtype=torch.int8, device=w.device)
    sc_loc = torch.zeros(rmax, dtype=torch.float32, device=w.device)
    it_loc = torch.zeros(rmax, dtype=torch.int32, device=w.device)
    if b > a:
        ops.ssz(w[a:b], s, bits, max_iters, q_loc[: b - a], sc_loc[: b - a], it_loc[: b - a])
    _gather_rows(q_loc, q_out, N, group)
    _gather_rows(sc_loc, scale_out, N, group)
    if iters_out is not None:
        _gather_rows(it_loc, iters_out, N, group)


def column_parallel_linear(x: torch.Tensor, inv_s: torch.Tensor | None, qw_shard: torch.Tensor,
                           sw_shard: torch.Tensor, y_shard: torch.Tensor, y_full: torch.Tensor | None = None,
                           group=None, ops=None) -> torch.Tensor:
    """The W8A8 linear of a layer whose output channels N are split across
    ranks (ColumnParallelLinear): every rank holds the whole x [M, K] and
    inv_s, and its block of the quantized weight, qw_shard [N_r, K] and
    sw_shard [N_r] (rows shard_rows(N, G, r), e.g. from ssz_quant_weight on
    those rows of W).  Each rank quantizes x per token (the same codes on
    every rank) and multiplies by its block: y_shard [M, N_r] = Y[:, N_r],
    with no exchange.  With y_full [M, N] given, the blocks are all-gathered
    into it on every rank.  Bit-identical to the unsharded linear."""
    ops = ops or KernelOps()
    M = x.shape[0]
    qx = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    sx = torch.empty(M, dtype=torch.float32, device=x.device)
    ops.quant_act(x, inv_s, qx, sx)
    if qw_shard.shape[0] > 0:
        ops.gemm(qx, sx, qw_shard, sw_shard, y_shard)
    if y_full is not None:
        G, N = world_size(group), y_full.shape[1]
        if G == 1:
            y_full.copy_(y_shard)
        else:
            rmax = -(-N // G)
            loc = torch.zeros(rmax, M, dtype=y_shard.dtype, device=y_shard.device)
            loc[: y_shard.shape[1]].copy_(y_shard.t())
            full_t = torch.empty(N, M, dtype=y_shard.dtype, device=y_shard.device)
            _gather_rows(loc, full_t, N, group)
            y_full.copy_(full_t.t())
    return y_shard


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
