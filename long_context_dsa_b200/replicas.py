"""Replica plumbing for the multi-GPU run: one process per GPU, launched by
torchrun, each running its own independent prefill (its own seeded sequence)
through the library.  The hot path has no exchange step -- every query's
indexer, top-k and attention read only its own sequence -- so there is no
data-path collective; the ranks meet only to start the timed region together
and to combine their device timings, the job's time being the slowest rank's.
"""

from __future__ import annotations


def rank_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic sequence (every rank draws different inputs)."""
    return base + rank


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of `x` over all ranks (the value itself without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return world * units_per_rank / (max_ms / 1e3)
