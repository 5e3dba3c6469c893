"""Data-parallel replicas: one process per GPU, each decoding its own batch of
sequences.  Caches, windows and queries are per sequence and the decode path has
no exchange step, so no collective touches the data: ranks only meet at
barriers and at the max-over-ranks step time.  Host-side helpers shared by the
benchmark and its multi-process tests (plumbing only; no method arithmetic)."""
from __future__ import annotations

from . import workloads as W

RANK_SEED_STRIDE = 1000  # rank r draws its sequences from seed + 1000 r


def rank_workload(base: W.Workload, rank: int) -> W.Workload:
    """The workload of rank `rank`: the same shapes, its own sequences."""
    return W.small(base, seed=base.seed + RANK_SEED_STRIDE * rank)


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """The largest x over all ranks (every rank gets it)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: the units every rank processed over the max-over-ranks time."""
    return units_per_rank * world / seconds
