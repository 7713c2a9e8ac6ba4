"""Host-side helpers for running the forward on several GPUs (one process per
GPU) with no data-path collective: every rank processes its own batch of
independent sequences (weak scaling).  The only collectives are the timing
barrier and max/sum reductions of scalars, which work on any torch.distributed
backend (NCCL on GPUs, gloo on CPU for tests).
"""
from __future__ import annotations

import torch


def _dist():
    import torch.distributed as dist
    return dist


def barrier(world: int) -> None:
    if world > 1:
        _dist().barrier()


def _reduce(x: float, world: int, op, device) -> float:
    if world == 1:
        return float(x)
    dist = _dist()
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def reduce_max(x: float, world: int, device="cpu") -> float:
    """Max of a per-rank scalar (the step time is the slowest rank's)."""
    return _reduce(x, world, _dist().ReduceOp.MAX if world > 1 else None, device)


def reduce_sum(x: float, world: int, device="cpu") -> float:
    """Sum of a per-rank scalar (tokens processed by all ranks)."""
    return _reduce(x, world, _dist().ReduceOp.SUM if world > 1 else None, device)


def rank_seed_offset(rank: int) -> int:
    """Seed offset of a rank's batch: ranks draw independent sequences."""
    return 1000 * int(rank)


def weak_scaling_throughput(tokens_all_ranks: float, ms_slowest_rank: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return tokens_all_ranks / (ms_slowest_rank * 1e-3)
