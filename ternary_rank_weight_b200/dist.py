"""Host-side plumbing for running independent factorizations on several GPUs.

Matrices are independent problems, so the work shards with no collective on
the data path: every rank factors its own matrices on its own device (one
process per GPU).  ``torch.distributed`` is used only for the barrier around a
timed region and for the max-over-ranks time (NCCL on GPUs, gloo on CPU).

A rank's matrices are the workload's shapes and recipe with seeds offset by
``rank * SEED_STRIDE`` (weak scaling: per-rank work is fixed as ranks are
added); ``partition`` / ``slice_workload`` instead split one fixed batch into
contiguous slices (strong scaling of a batch: the total work stays fixed).
"""
from __future__ import annotations

import os
from dataclasses import dataclass, replace

import torch

SEED_STRIDE = 1000


@dataclass(frozen=True)
class RankInfo:
    world: int
    rank: int
    local: int


def rank_info() -> RankInfo:
    """World size, rank and local rank from the launcher's environment (1, 0, 0 if unset)."""
    return RankInfo(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def rank_seeds(seeds, rank: int):
    """Seeds of this rank's matrices: the workload's seeds offset by rank * SEED_STRIDE."""
    return tuple(int(s) + SEED_STRIDE * rank for s in seeds)


def rank_workload(workload, rank: int):
    """The workload a rank factors under weak scaling (same shapes, own seeds)."""
    return replace(workload, seeds=rank_seeds(workload.seeds, rank))


def slice_workload(workload, world: int, rank: int):
    """This rank's contiguous slice of a batch (strong scaling): the same matrices (same seeds)
    as in the whole batch.  Returns (sliced workload, indices into the batch)."""
    idx = partition(workload.count, world, rank)
    pick = lambda t: tuple(t[i] for i in idx)   # noqa: E731
    return replace(workload, shapes=pick(workload.shapes), seeds=pick(workload.seeds), mu=pick(workload.mu),
                   tau=pick(workload.tau)), idx


def partition(count: int, world: int, rank: int) -> range:
    """Contiguous slice of ``count`` items for ``rank``: sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    lo = (count * rank) // world
    hi = (count * (rank + 1)) // world
    return range(lo, hi)


def max_over_ranks(x: float, device=None) -> float:
    """The largest of every rank's ``x`` (the rank's own value when not distributed)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    """Sum of every rank's ``x``."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None) -> None:
    """Barrier over ranks (if distributed), then wait for this rank's device work."""
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()
    if device is not None and getattr(device, "type", None) == "cuda":
        torch.cuda.synchronize(device)


def throughput(units_all_ranks: float, t_ms_max: float) -> float:
    """Whole-job rate: units processed by all ranks divided by the slowest rank's time."""
    if t_ms_max <= 0:
        raise ValueError("time must be positive")
    return units_all_ranks / (t_ms_max / 1000.0)
