"""Data-parallel replicas of the pruned-MLP block across GPUs of one node.

Samples are independent (the MLP acts on each token alone, and top-k is per
sample), so N GPUs run N independent replicas: rank r takes its own batch (seed
base + r) and nothing is exchanged on the data path. The only collectives are
host-side bookkeeping: a barrier around timed regions and a max over ranks of
the elapsed time (the job finishes when the slowest rank does).
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch
import torch.distributed as dist


def env_ranks() -> Tuple[int, int, int]:
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 if absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> Tuple[int, int, int]:
    """Joins the process group when WORLD_SIZE > 1 (short timeout: a missing rank ends
    the next collective with an error instead of waiting for ever)."""
    world, rank, local = env_ranks()
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank's shard: every replica draws a different batch of the same shape."""
    return base_seed + rank


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(value: float, world: int, device: torch.device | None = None) -> float:
    """The largest `value` over all ranks (the job's elapsed time)."""
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, steps: int, max_total_ms: float, world: int) -> float:
    """Whole-job tokens/s: every rank processes its own tokens; the job takes as long
    as its slowest rank (weak scaling)."""
    if max_total_ms <= 0:
        raise ValueError("elapsed time must be positive")
    return world * tokens_per_rank_step * steps / (max_total_ms / 1e3)


def shutdown(world: int) -> None:
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
