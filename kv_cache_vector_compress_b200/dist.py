"""Host-side multi-GPU plumbing: one process per GPU, independent work per rank.

The compression path partitions into independent (batch, KV-head) slices, so ranks share no data
and no collective runs on the data path.  The only collective is the timing reduction: the
reported time of a timed region is the maximum over ranks.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local: int


def rank_info() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> RankInfo:
    """Join the process group when launched with more than one rank (torchrun env)."""
    ri = rank_info()
    if ri.world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return ri


def barrier():
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device: str | torch.device = "cpu") -> float:
    """Max of a scalar over all ranks (identity with one rank)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def seed_offset(rank: int) -> int:
    """Per-rank offset of the input seeds: each rank compresses and attends its own batch."""
    return 7919 * rank


def shard(n: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [start, start + count) share of n independent units for this rank (the first
    n % world ranks take one extra unit)."""
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def weak_scaling_value(units_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / max_seconds


def destroy():
    if dist.is_initialized():
        dist.destroy_process_group()
