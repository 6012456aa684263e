"""Data-parallel plumbing for running the layer on several GPUs of one node.

The W4.4A8 linear layer shards without any exchange: every rank holds the
same packed weights and processes its own batch of tokens (the tokens of a
batch are independent rows of X).  The only collectives are host-side
bookkeeping -- a barrier around timed regions and the max of the ranks'
device times -- never on the data path.  These helpers work with any
torch.distributed backend (NCCL on GPUs, gloo on CPU for the tests).
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
    local_rank: int


def rank_info() -> RankInfo:
    """Rank, world size and local rank from the launcher's environment."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device=None) -> RankInfo:
    """Initialise the default process group when more than one rank runs."""
    info = rank_info()
    if info.world > 1 and not dist.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)
    return info


def batch_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s activation batch: distinct per rank, so the ranks
    process different tokens (weak scaling: a fixed batch per GPU)."""
    return base_seed + rank


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar (e.g. a device-measured time) over all ranks."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_rows(m_total: int, rank: int, world: int) -> tuple:
    """Token rows [start, stop) of a global batch of `m_total` rows that rank
    `rank` of `world` takes: contiguous shards whose sizes differ by at most
    one, the larger ones first (strong scaling: a fixed batch split over GPUs)."""
    base, extra = divmod(m_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def gather_rows(local: torch.Tensor, m_total: int, world: int) -> torch.Tensor:
    """The ranks' row shards (as cut by shard_rows) put back together in rank
    order on every rank.  Shards are padded to the largest for all_gather."""
    if world == 1:
        return local
    if local.element_size() < 4:  # narrow types go through int32 (not every backend gathers them)
        narrow = {1: torch.int8, 2: torch.int16}[local.element_size()]
        wide = gather_rows(local.view(narrow).to(torch.int32), m_total, world)
        return wide.to(narrow).view(local.dtype)
    rows = [shard_rows(m_total, r, world) for r in range(world)]
    width = max(stop - start for start, stop in rows)
    pad = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([parts[r][:stop - start] for r, (start, stop) in enumerate(rows)])


def total_units(units_per_rank: int, world: int) -> int:
    """Work done by the whole job when each rank processes `units_per_rank`."""
    return units_per_rank * world


def shutdown(world: int) -> None:
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
