"""Process-group plumbing for running the TTQ path on several GPUs of one node.

The TTQ hot path partitions by prompt: each prompt has its own statistic s and its own
codes, so N GPUs run N independent prompt streams (weak scaling) with no data-path
collective. torch.distributed is used only to line the ranks up (a barrier) and to
take the slowest rank's time (an all-reduce of one number).
"""

from __future__ import annotations

import datetime
import os


def env():
    """(rank, world_size, local_rank) from the torchrun environment (defaults 0, 1, 0)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init(backend: str, timeout_s: float = 120.0):
    """Initialises the default process group when WORLD_SIZE > 1; returns world size."""
    import torch.distributed as dist

    rank, world, _ = env()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return world


def shard(n_units: int, rank: int, world: int):
    """Contiguous share [lo, hi) of n_units for one rank (sizes differ by at most one)."""
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's own synthetic prompts (rank 0 keeps the workload's seed)."""
    return base_seed + 7919 * rank


def barrier():
    import torch.distributed as dist

    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (the value itself on a single process)."""
    import torch
    import torch.distributed as dist

    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def finalize():
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()
