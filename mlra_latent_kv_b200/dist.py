"""Multi-GPU plumbing for the decode benchmark: one process per GPU.

Decode over a batch of independent sequences shards by sequence with no
exchange at all, so N GPUs run N replicas of the step, each on its own batch
(weak scaling).  The only collectives are the timing barrier and the
max-over-ranks reduction of the measured time; nothing on the data path.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def world() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0) -> bool:
    """Joins the process group when launched with more than one rank."""
    _, ws, _ = world()
    if ws <= 1 or dist.is_initialized():
        return dist.is_initialized()
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return True


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank r's batch: each replica decodes different sequences."""
    return seed + 1000 * rank


def barrier(device=None):
    if dist.is_initialized():
        if dist.get_backend() == "nccl" and device is not None:
            dist.barrier(device_ids=[torch.device(device).index])
        else:
            dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    if not dist.is_initialized():
        return float(x)
    dev = device if (device is not None and dist.get_backend() == "nccl") else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(units_per_rank: float, world_size: int, max_seconds: float) -> float:
    """Whole-job rate: units processed by all ranks over the slowest rank's time."""
    return units_per_rank * world_size / max_seconds


def shutdown():
    if dist.is_initialized():
        dist.destroy_process_group()
