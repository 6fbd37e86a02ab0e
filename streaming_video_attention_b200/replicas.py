"""Several GPUs, one process each, running the warmup path as independent replicas.

The path has no exchange step: every sequence (its KV cache, its statistics, its absorb
solve and layer selection [ISPA §3.1, §3.3]) belongs to one stream of video, so N GPUs run
N independent episodes and no collective touches the data path. What crosses ranks is only
the bookkeeping here: a barrier around the timed region and the maximum of the ranks'
device times. Throughput is the units every rank processed over the slowest rank's time
(weak scaling: the per-rank work is fixed as N grows).
"""
from __future__ import annotations

import dataclasses
import os
from typing import Tuple

import torch
import torch.distributed as dist


def world() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def _multi() -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1


def barrier() -> None:
    if _multi():
        dist.barrier()


def slowest(seconds: float, device="cpu") -> float:
    """Maximum of `seconds` over all ranks (every rank must call it, in the same order)."""
    t = torch.tensor([float(seconds)], dtype=torch.float64, device=device)
    if _multi():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, seconds: float, device="cpu") -> Tuple[float, float]:
    """(units of the whole job per second, slowest rank's seconds)."""
    n = dist.get_world_size() if _multi() else 1
    t = slowest(seconds, device)
    return n * float(units_per_rank) / t, t


def replica_config(cfg, rank: int):
    """The workload of replica `rank`: same shapes, its own seed (distinct input streams)."""
    return dataclasses.replace(cfg, seed=int(cfg.seed) + 7919 * int(rank))
