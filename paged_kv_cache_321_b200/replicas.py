"""Multi-GPU operation: independent replicas.

The paged KV cache hot path shards by request with no exchange between GPUs:
each rank owns its pool, its block tables and its sequences, and runs the
same kernels. torch.distributed (NCCL on GPUs, gloo on CPU) is used only for
start-up, barriers and the max-over-ranks reduction of timings; no tensor of
the data path crosses GPUs.
"""

from __future__ import annotations

import datetime
import os
from typing import Sequence


def world_from_env():
    """(rank, world_size, local_rank) from the torchrun environment."""
    if "RANK" not in os.environ:
        return 0, 1, 0
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    return rank, world, int(os.environ.get("LOCAL_RANK", rank))


def init(backend: str, timeout_s: float = 120.0, device=None):
    """Initialises the default process group (short timeout, so ranks that
    wait for one another end with an error rather than hang)."""
    import torch.distributed as dist

    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return dist


def replica_seed_offset(base_offset: int, rank: int) -> int:
    """Seed offset of rank `rank`'s replica: every rank draws its own
    requests, so ranks never process identical inputs."""
    return base_offset + 1000 * rank


def max_over_ranks(values: Sequence[float], dist=None, device=None) -> list:
    """Element-wise maximum of per-rank values (timings) over all ranks."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes
    units_per_rank; the job takes as long as its slowest rank."""
    return units_per_rank * world / seconds_max
