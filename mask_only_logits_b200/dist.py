"""Multi-process plumbing (one process per GPU, torch.distributed): rank discovery, timing
reduced as the maximum over ranks, and contiguous sharding of a range across ranks.

The decode step of independent batches shares nothing, so ``bench.py`` runs one replica
per rank (weak scaling) and only reduces timings; ``shard_range`` splits a range (e.g. the
vocabulary) into contiguous per-rank pieces for callers that shard one problem.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info() -> RankInfo:
    """RANK / WORLD_SIZE / LOCAL_RANK from the environment (torchrun's), defaults 0/1/0."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init_process_group(backend: str, timeout_s: float = 120.0, device: torch.device | None = None):
    """Initialise the default process group from the environment with a short timeout (so
    that ranks waiting on a rank that died end with an error instead of hanging)."""
    import torch.distributed as dist
    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if device is not None and device.type == "cuda":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return dist


def max_over_ranks(values, device: torch.device | None = None) -> list[float]:
    """Element-wise maximum of a list of floats over all ranks (identity without a group)."""
    import torch.distributed as dist
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device or torch.device("cpu"))
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def sum_over_ranks(values, device: torch.device | None = None) -> list[float]:
    """Element-wise sum of a list of floats over all ranks (identity without a group)."""
    import torch.distributed as dist
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device or torch.device("cpu"))
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.cpu()]


def shard_range(total: int, rank: int, world: int) -> tuple[int, int]:
    """[lo, hi) of rank's contiguous share of range(total): sizes differ by at most one and
    the shares tile the range in rank order."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    return total * rank // world, total * (rank + 1) // world


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of rank's replica of a synthetic workload (distinct batches per rank)."""
    return base_seed + rank
