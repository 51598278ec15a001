"""Host-side multi-rank helpers (one process per GPU, torch.distributed).

The hot path shards by sequence: every rank compresses its own sequences and
decodes its own caches, so there is no collective on the data path.  Ranks only
meet to agree on timing: every timed quantity is reduced with MAX over ranks
(a step is as slow as its slowest rank).
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def rank_info():
    """(rank, local_rank, world_size) from the torchrun environment (1 process if unset)."""
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic inputs: disjoint streams per rank."""
    return int(base_seed) + 100 * int(rank)


def shard_range(n_units: int, rank: int, world: int):
    """Contiguous [begin, end) share of n_units for a rank (sizes differ by at most 1)."""
    base, extra = divmod(int(n_units), int(world))
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def max_over_ranks(values, device=None):
    """Element-wise MAX of a list of floats over all ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank: float, world: int, max_time_s: float) -> float:
    """Aggregate throughput: the units all ranks processed over the slowest rank's time."""
    return world * float(units_per_rank) / float(max_time_s)


def tsp_exchange_raw(raw_local: torch.Tensor, group=None) -> torch.Tensor:
    """The one exchange step of head-sharded token-selective propagation
    (FastKV section 2.A: saliency aggregated over all heads of the layer).

    raw_local is this rank's [n_local, S] float32 raw window scores (its KV
    heads; every rank holds the same n_local).  It is summed element-wise
    over the ranks in place (all-reduce, SUM) and returned: the TSP step then
    adds its n_local rows, which gives the sum over every head of the layer,
    and every rank selects the same token set.  Without a process group the
    tensor is returned unchanged.  The addition order differs from one
    device's, so equal-up-to-rounding scores may tie-break differently (the
    selection agrees outside the 1e-5 tie band)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(raw_local, op=dist.ReduceOp.SUM, group=group)
    return raw_local
