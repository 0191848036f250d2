"""Host logic of data-parallel replicas: one process per GPU, each running the whole
forward on its own images.

The tower's images are independent and the vision encoder is loaded whole on every
rank, so the forward needs no collective; ranks exchange only timings (a max
reduction) and synchronise with barriers.  These helpers hold that logic so that the
benchmark and the tests share it; they work with any torch.distributed backend
(NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import os


def rank_env() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (defaults 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def split_batch(global_batch: int, world: int, rank: int) -> tuple[int, int]:
    """(first image, image count) of this rank when a global batch is shared out:
    contiguous shares whose sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world or global_batch < 0:
        raise ValueError("bad world/rank/batch")
    base, extra = divmod(global_batch, world)
    count = base + (1 if rank < extra else 0)
    first = rank * base + min(rank, extra)
    return first, count


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic images (weights use the base seed on every rank)."""
    return base_seed + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank value over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_per_step: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return world * units_per_rank_per_step * steps / (max_ms / 1000.0)
