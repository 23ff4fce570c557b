"""Shot sharding over the ranks of one process group.

Shots are independent, so a run over several GPUs gives each rank (one
process per GPU) a contiguous block of shots with the model replicated; the
only exchange is the sum of the model gradients over ranks (one all-reduce
per gradient field), and device times are reported as the maximum over
ranks.  The functions work with any torch.distributed backend (NCCL on GPUs,
gloo on CPU tensors) and are no-ops in a single-process run.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shot_block(n_total: int, rank: int, world: int) -> tuple[int, int]:
    """[lo, hi) of the shots owned by `rank`: contiguous blocks whose sizes
    differ by at most one, covering 0 .. n_total - 1 exactly once."""
    if world < 1 or not 0 <= rank < world or n_total < 0:
        raise ValueError("bad rank / world / shot count")
    base, extra = divmod(n_total, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def _active() -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1


def sum_over_ranks_(*tensors: torch.Tensor) -> None:
    """In-place sum of each tensor over all ranks (the gradient exchange)."""
    if not _active():
        return
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank scalar (a device time) over all ranks."""
    if not _active():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
