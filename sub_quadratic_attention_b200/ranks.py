"""Host-side logic of a multi-GPU run (one process per GPU, torch.distributed).

The mix shards over the batch: every rank mixes its own independent batch of
the workload, so no data crosses GPUs.  What the ranks share is only the
timing: each rank times its own steps on the device, the job's time is the
maximum over ranks, and the job's throughput is the tokens of all ranks over
that time (weak scaling: the work per rank is fixed as ranks are added).
"""
from __future__ import annotations

from typing import Optional

import torch


def rank_seed_offset(rank: int) -> int:
    """Seed offset of a rank's batch: rank r draws its inputs with seed + r."""
    return int(rank)


def max_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """Maximum of `value` over all ranks of the default process group (the
    value itself when torch.distributed is not initialised).  With the NCCL
    backend pass the rank's CUDA device; gloo reduces on the CPU."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, world: int, steps: int, max_total_ms: float) -> float:
    """Whole-job tokens per second: all ranks' tokens over the slowest rank's time."""
    if steps <= 0 or max_total_ms <= 0:
        raise ValueError("steps and time must be positive")
    return tokens_per_rank_step * world * steps / (max_total_ms * 1e-3)
