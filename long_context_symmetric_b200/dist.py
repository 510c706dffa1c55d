"""Process-per-GPU plumbing for running the hot path on several GPUs.

The Lighthouse path partitions into independent (batch, head) problems: the
selection, the sub-sequence and its attention are all per head ("Long Context
Pre-Training with Lighthouse Attention", Fig. 2: the index set has shape
[B, H, K]). So N GPUs run N replicas, each on its own batch rows, with no
collective on the data path (weak scaling: per-GPU work fixed). The only
collectives are for measurement: a barrier around the timed region and the
max over ranks of the device time.
"""

from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist

__all__ = ["RankInfo", "rank_info", "init", "replica_seed", "batch_rows", "max_over_ranks",
           "barrier", "job_throughput", "shutdown"]


class RankInfo:
    def __init__(self, rank: int, world: int, local: int):
        self.rank, self.world, self.local = rank, world, local

    def __repr__(self):
        return f"RankInfo(rank={self.rank}, world={self.world}, local={self.local})"


def rank_info() -> RankInfo:
    """Rank, world size and local rank from the torchrun environment (1 process if absent)."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", device: torch.device | None = None, timeout_s: float = 120.0) -> bool:
    """Join the process group when WORLD_SIZE > 1; returns whether a group exists.

    A short timeout makes ranks that wait on a missing peer end with an error.
    """
    info = rank_info()
    if info.world <= 1:
        return False
    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if backend == "nccl" and device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return True


def replica_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s own batch (distinct per rank, reproducible)."""
    return seed + 101 * rank


def batch_rows(global_batch: int, rank: int, world: int) -> range:
    """Rows of a global batch that rank `rank` processes (contiguous, balanced)."""
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def barrier():
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """Max of a per-rank scalar (the timed region's device milliseconds) over all ranks."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job rate: the units all ranks processed divided by the slowest rank's time."""
    return units_per_rank * world / seconds_max


def shutdown():
    if dist.is_initialized():
        dist.destroy_process_group()
