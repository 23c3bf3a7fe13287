"""Data-parallel plumbing for multi-GPU runs (one process per GPU).

Decode over the compressed cache shards by sequence: every sequence's cache,
indexer scan, top-K and attention are independent, so N ranks simply decode
N disjoint batches (replicas; weak scaling) and no collective touches the
data path.  The only cross-rank steps are host-side: a barrier around the
timed region and a MAX reduction of the per-rank device time, so the
reported throughput is whole-job work over the slowest rank's time.
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist

SEED_STRIDE = 1000


def world() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_workload(w, rank: int):
    """The workload a rank decodes: same shapes, its own sequences (seed)."""
    return w.scaled(seed=w.seed + SEED_STRIDE * rank)


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """MAX of a per-rank scalar (device time in ms) across the job."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(steps: int, batch_per_rank: int, world_size: int, ms_max: float) -> float:
    """Query tokens per second of the whole job: every rank advances its
    batch_per_rank sequences by `steps` tokens; the job takes the slowest
    rank's time."""
    return steps * batch_per_rank * world_size / (ms_max / 1e3)
