"""Data-parallel plumbing for calibration across ranks (one process per GPU).

Calibration is a per-channel maximum over a token stream, so ranks that
each calibrate on their own shard of tokens merge exactly with an
element-wise MAX all-reduce of the [K] maxima (order-free, bit-exact).  The
linear itself needs no exchange: every rank holds the same smoothed INT8
weights and quantizes its own tokens.
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
