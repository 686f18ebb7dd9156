"""Data-parallel plumbing for the smoothed W8A8 linear (one process per GPU).

The online path has no exchange: each rank quantises and multiplies its own tokens against a
replica of the INT8 weight. Calibration has one: each rank reduces its own share of the calibration
tokens to a per-channel abs-max, and the shares are combined with an all-reduce(MAX) of the fp32 [K]
vector before the smoothing factors are computed. The maximum is order-free, so the sharded result is
bit-identical to the unsharded one.
"""
from __future__ import annotations

import os
from typing import Callable, Iterable, Optional, Tuple

import torch
import torch.distributed as dist


def env_rank() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (0, 0, 1 when absent)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def shard_range(total: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) share of ``total`` units for ``rank`` (shares differ by at most 1)."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_max_(t: torch.Tensor, group=None) -> torch.Tensor:
    """In-place all-reduce(MAX) across the process group (no-op when not initialised / world 1)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t


def sharded_absmax(batches: Iterable, absmax_fn: Callable, init: Optional[torch.Tensor] = None,
                   group=None) -> torch.Tensor:
    """Running abs-max over this rank's calibration batches, then combined across ranks.

    absmax_fn(batch, amax_or_None) -> amax: the per-rank reduction (the libsq kernel on a GPU).
    """
    amax = init
    for b in batches:
        amax = absmax_fn(b, amax)
    if amax is None:
        raise ValueError("no calibration batch on this rank")
    return allreduce_max_(amax, group)
