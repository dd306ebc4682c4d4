"""Host-side logic of the multi-GPU benchmark (weak scaling, no collective on
the data path).

Every rank runs an independent batch of the same shape (work units of
different ranks never exchange data); the job's throughput is all ranks' work
over the slowest rank's device time.  The only collectives are the barrier
around the timed region and the max-reduction of the timings, both on the
host-visible process group (NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

import os


def rank_env():
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's independent batch (rank 0 uses the workload's own seed)."""
    return int(base_seed) + int(rank)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_step_per_rank: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank's flops over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("elapsed time must be positive")
    return flops_per_step_per_rank * world * steps / (max_ms * 1e-3) / 1e12
