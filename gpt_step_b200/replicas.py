"""Host logic of the multi-GPU mode: one independent replica of the step per rank.

The training step has no exchange between GPUs here; each rank trains its own
replica on its own token stream (weak scaling). What the ranks share is the
measurement: the job's time is the slowest rank's, and its throughput counts
every rank's tokens. The data-parallel arrangement of "Pretraining and adapting
a language model on a dependency-free stack" (§4.4: one gradient exchange per
optimizer step across the cards) is what these replicas stand in for.
"""
from __future__ import annotations

import os


def rank_env() -> tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(base: int, rank: int) -> int:
    """Seed of a rank's replica: its weights and its token stream differ from every other rank's."""
    return base + rank


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks of the default process group (any
    backend); the value itself when there is no group or only one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max / 1000.0)
