"""Multi-GPU plumbing (one process per GPU).

Calibration is a per-channel maximum over a token stream, so ranks that
each calibrate on their own shard of tokens merge exactly with an
element-wise MAX all-reduce of the [K] maxima (order-free, bit-exact).  A
data-parallel linear needs no exchange: every rank holds the same smoothed
INT8 weights and quantizes its own tokens.

A column-parallel linear splits the output channels: rank r holds the rows
[n0, n1) of Wq and w_scale and computes Y[:, n0:n1].  The full Y is then
either gathered (an all-gather of the shards) or, when every rank can store
into the others' Y buffers (peer-mapped memory), written straight into all
of them by the GEMM's own epilogue (sq_w8a8_linear_scatter), after which a
barrier on the stream orders the peers' writes before Y is used.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(total: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of `rank`'s contiguous share of `total` items; the first
    total % world ranks take one extra item."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_amax(amax: torch.Tensor, group=None) -> torch.Tensor:
    """In place: amax <- element-wise max of every rank's amax."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def column_shard(n: int, world: int, rank: int, align: int = 16) -> tuple[int, int]:
    """[n0, n1) of `rank`'s output channels: N split into blocks of `align`
    (the GEMM's column granularity) shared out as evenly as shard_range does."""
    if n % align != 0:
        raise ValueError(f"N={n} is not a multiple of {align}")
    b0, b1 = shard_range(n // align, world, rank)
    return b0 * align, b1 * align


def column_parallel_linear(xq: torch.Tensor, x_scale: torch.Tensor, wq_shard: torch.Tensor,
                           w_scale_shard: torch.Tensor, n_total: int, out_dtype=torch.bfloat16, group=None,
                           peers=None, linear=None) -> torch.Tensor:
    """Y [M, n_total] of a column-parallel linear on every rank.

    wq_shard / w_scale_shard are this rank's rows column_shard(n_total, world,
    rank) of Wq / w_scale.  With `peers` -- every rank's full Y tensor as this
    rank can address it (its own at index `rank`), all of them of dtype
    out_dtype -- the GEMM writes its shard into all of them and a one-element
    all-reduce on the stream orders every rank's writes before returning this
    rank's Y.  Without, the shards are all-gathered (padded to the widest
    shard) and reassembled.  `linear(xq, x_scale, wq, w_scale, out_dtype)`
    computes one shard (sq_w8a8_linear unless given)."""
    from . import sq_w8a8_linear, sq_w8a8_linear_scatter

    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    n0, n1 = column_shard(n_total, world, rank)
    if wq_shard.shape[0] != n1 - n0:
        raise ValueError("wq_shard does not hold this rank's column shard")
    M = xq.shape[0]
    if peers is not None:
        if len(peers) != world:
            raise ValueError("one peer tensor per rank")
        if n1 > n0:
            sq_w8a8_linear_scatter(xq, x_scale, wq_shard, w_scale_shard, list(peers), n0)
        if world > 1:
            token = torch.zeros(1, device=xq.device)
            dist.all_reduce(token, group=group)  # every rank's stores precede this on its stream
        return peers[rank]
    linear = linear or sq_w8a8_linear
    if n1 > n0:
        y_local = linear(xq, x_scale, wq_shard, w_scale_shard, out_dtype)
    else:  # more ranks than 16-column blocks: this rank holds nothing
        y_local = torch.empty((M, 0), dtype=out_dtype, device=xq.device)
    if world == 1:
        return y_local
    widths = [column_shard(n_total, world, r)[1] - column_shard(n_total, world, r)[0] for r in range(world)]
    wmax = max(widths)
    send = torch.zeros((M, wmax), dtype=y_local.dtype, device=y_local.device)
    send[:, :n1 - n0] = y_local
    recv = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(recv, send, group=group)
    return torch.cat([recv[r][:, :widths[r]] for r in range(world)], dim=1)

