"""Host-side multi-GPU plumbing: one process per GPU, independent work per rank.

The compression path partitions into independent (batch, KV-head) slices, so ranks share no data
and no collective runs on the data path; the timing reduction (the reported time of a timed
region is the maximum over ranks) is the only collective there.  Two paths have one real exchange
each: vector search over a database sharded across ranks gathers every rank's top-k list of each
query and merges them (sharded_topk); attention over one long context split across ranks gathers
each rank's (max, sum, weighted value sum) partial of its token range and merges them
(sharded_attend).
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


def merge_topk(vals: torch.Tensor, idx: torch.Tensor, k: int):
    """The k best of candidate lists [..., n] (score, key index) in the order of the top-k step:
    score descending, ties to the smaller index.  Returns (idx, vals) [..., k]."""
    o = torch.argsort(idx, dim=-1, stable=True)
    v1, i1 = vals.gather(-1, o), idx.gather(-1, o)
    o2 = torch.argsort(v1, dim=-1, descending=True, stable=True)
    return i1.gather(-1, o2)[..., :k], v1.gather(-1, o2)[..., :k]


def sharded_topk(local_idx: torch.Tensor, local_val: torch.Tensor, k: int, offset: int):
    """Global top-k of a database sharded over the ranks.  Each rank passes the top-k of its own
    shard (indices local to the shard, which starts at key `offset`); the lists are gathered from
    all ranks (one all_gather each for indices and scores) and merged.  Every rank returns the
    global (idx, vals) [..., k]."""
    gidx = local_idx.to(torch.int64) + offset
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return merge_topk(local_val, gidx, k)
    world = dist.get_world_size()
    all_v = [torch.empty_like(local_val) for _ in range(world)]
    all_i = [torch.empty_like(gidx) for _ in range(world)]
    dist.all_gather(all_v, local_val.contiguous())
    dist.all_gather(all_i, gidx.contiguous())
    return merge_topk(torch.cat(all_v, dim=-1), torch.cat(all_i, dim=-1), k)


def context_shard(T: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous token range [start, start + count) of a T-token context that this rank attends
    when one long context is split across the ranks."""
    return shard(T, world, rank)


def gather_partials(partial: torch.Tensor) -> torch.Tensor:
    """All ranks' attention partials [..., dim + 2] stacked in rank order: [world, ...] (one
    all_gather; every rank receives all of them)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return partial.unsqueeze(0)
    world = dist.get_world_size()
    parts = [torch.empty_like(partial) for _ in range(world)]
    dist.all_gather(parts, partial.contiguous())
    return torch.stack(parts)


def sharded_attend(p, q: torch.Tensor, keys, values, Hkv: int, T_local: int, scale: float = 0.0):
    """Attention over a long context split across the ranks: every rank holds the packed keys and
    values of its own token range (context_shard) and the same queries; it computes the partial of
    its range (tq_attend_partial), the partials are all-gathered, and each rank merges them
    (tq_attend_merge: log-sum-exp of the pieces, then the single rotation back).  Returns the
    attention output [B, Hq, Nq, dim] on every rank."""
    from . import tq
    part = tq.tq_attend_partial(p, q, keys, values, Hkv, T_local, scale=scale)
    return tq.tq_attend_merge(p, gather_partials(part))


def destroy():
    if dist.is_initialized():
        dist.destroy_process_group()
