"""Host-side logic of the multi-GPU path.

Heads are independent and each keeps its own state, so a job spreads over
ranks (one process per GPU) by heads, with no collective on the data path:
rank r runs its own contiguous range of heads, or, in the weak-scaling
benchmark, its own replica of the workload. The only collectives are the
timing reduction (device time, max over ranks) and, where a caller wants every
head on one rank, a gather of the results.
"""
from __future__ import annotations


def head_range(n_heads: int, world: int, rank: int) -> tuple[int, int]:
    """[lo, hi) of the heads rank `rank` owns when `n_heads` heads are split over
    `world` ranks: contiguous, sizes differing by at most one, earlier ranks
    taking the extra heads."""
    if world < 1 or not 0 <= rank < world or n_heads < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, n_heads >= 0")
    base, extra = divmod(n_heads, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks of the default process group (the
    value itself without one). `device` is where the reduction tensor lives:
    a CUDA device for NCCL, None (CPU) for gloo."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Units per second for the whole job: every rank processed `units_per_rank`
    units per step, and the slowest rank took `max_ms` for all steps."""
    if max_ms <= 0:
        raise ValueError("max_ms must be positive")
    return units_per_rank * steps * world / (max_ms / 1e3)
