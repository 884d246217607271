"""Host-side logic of the multi-GPU (one process per GPU) runs.

Every row (batch entry, KV head) of the decode step is independent: its
attention, score, argmin and eviction read only that row.  So N GPUs take N
independent batches (weak scaling) and no collective is needed on the data
path; the only collectives are the barrier before the timed region and the
max over ranks of the measured time.
"""
from __future__ import annotations

from typing import Sequence

from .synth import DecodeConfig


def rank_config(cfg: DecodeConfig, rank: int) -> DecodeConfig:
    """The workload rank `rank` runs: same shapes and recipe, its own seed."""
    return cfg if rank == 0 else cfg.with_(seed=cfg.seed + 1000 * rank)


def shard_batch(batch: int, world: int, rank: int) -> Sequence[int]:
    """Batch entries of `rank` when one batch is split over `world` ranks
    (contiguous blocks; the first `batch % world` ranks take one more)."""
    base, extra = divmod(batch, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, device=None) -> float:
    """Max of `value` over all ranks of the default process group (the time
    of the slowest rank); `value` itself when not distributed."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps_per_rank: int, max_ms: float) -> float:
    """Units all ranks processed divided by the slowest rank's time."""
    return world * steps_per_rank / (max_ms / 1e3)
