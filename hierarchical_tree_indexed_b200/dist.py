"""Multi-GPU plumbing of the decode benchmark: one process per GPU.

The path shards by (sequence, KV head): trees, routing and attention of
different sequences share nothing, so each rank owns whole sequences and the
data path has no collective.  The only cross-rank steps are a barrier around
the timed region and the max of the ranks' device times.
"""
from __future__ import annotations

import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Rank:
    rank: int = 0
    world: int = 1
    local: int = 0

    @property
    def leader(self) -> bool:
        return self.rank == 0


def from_env() -> Rank:
    return Rank(int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
                int(os.environ.get("LOCAL_RANK", 0)))


def init(r: Rank, backend: str = "nccl", timeout_s: float = 120.0) -> None:
    if r.world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, rank=r.rank, world_size=r.world,
                                timeout=datetime.timedelta(seconds=timeout_s))


def shard(total: int, r: Rank) -> range:
    """Contiguous share of `total` units (sequences) for rank r; shares differ by at most one."""
    base, extra = divmod(total, r.world)
    start = r.rank * base + min(r.rank, extra)
    return range(start, start + base + (1 if r.rank < extra else 0))


def barrier(r: Rank, device=None) -> None:
    if r.world > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x: float, r: Rank, device=None) -> float:
    """Max of a per-rank scalar (device times are combined this way)."""
    if r.world == 1:
        return float(x)
    dev = device if (device is not None and dist.get_backend() == "nccl") else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, r: Rank, device=None) -> float:
    if r.world == 1:
        return float(x)
    dev = device if (device is not None and dist.get_backend() == "nccl") else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def finish(r: Rank) -> None:
    if r.world > 1 and dist.is_initialized():
        dist.destroy_process_group()
