"""Multi-GPU plumbing: one process per GPU, torch.distributed for the host side.

Trajectories are independent, so an ensemble shards into contiguous blocks of
trajectories with no exchange on the data path.  The one quantity that spans
trajectories is the d = 64 system's weight gradient dL/dW = sum_i dL_i/dW: when
one ensemble is split across ranks, each rank's gs_grad returns the sum over
its shard and a sum all-reduce of the 64 x 64 matrix (16 KB in fp32) completes
it.  Benchmarks time each rank on the device and take the maximum over ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard(n_total: int, rank: int, world: int) -> tuple[int, int]:
    """(start, count) of rank's contiguous block of n_total trajectories;
    blocks differ in size by at most one and cover every trajectory once."""
    if world < 1 or not 0 <= rank < world or n_total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n_total, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def allreduce_shared_grad(dshared: torch.Tensor) -> torch.Tensor:
    """Sum the per-rank weight gradients in place (no-op on a single rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(dshared, op=dist.ReduceOp.SUM)
    return dshared


def max_over_ranks(values, device=None) -> list[float]:
    """Element-wise maximum over ranks of a list of floats (e.g. timings)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()
