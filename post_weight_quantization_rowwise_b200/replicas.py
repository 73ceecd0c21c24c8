"""Host-side plumbing for running the quantizer on several GPUs, one process each.

Rows, tensors and experts are independent problems, so nothing on the data path
crosses ranks: each rank quantizes its own units with the same kernels.  What
does cross ranks is bookkeeping:

* ``shard``: a contiguous, balanced partition of a list of units (for example
  the tensors of a model) over the ranks;
* ``rank_seed_offset``: distinct synthetic inputs per rank for weak scaling;
* ``max_over_ranks``: the job time of a timed region (the slowest rank);
* ``sum_over_ranks``: the job's totals (values processed, bytes copied), so that
  a rate is all ranks' work over the slowest rank's time;
* ``reduce_rmse``: the weighted-RMSE accumulators of all ranks combined
  (sums added, ``max|e|`` maxed), so that one tensor set split over ranks gives
  the same statistics as on one rank (up to binary64 rounding order);
* ``job_rmse``: the job's round-trip statistics from every rank's accumulator and
  value count (what the benchmark reports for several GPUs).

The functions take an initialised ``torch.distributed`` process group (NCCL on
GPUs, gloo on CPU) or work on one process when none is initialised.
"""
from __future__ import annotations

from typing import Sequence, TypeVar

T = TypeVar("T")

SEED_STRIDE = 1_000_000


def rank_seed_offset(rank: int) -> int:
    return SEED_STRIDE * int(rank)


def shard(units: Sequence[T], rank: int, world: int) -> list[T]:
    """Contiguous block of ``units`` for ``rank``; sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    n = len(units)
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return list(units[start:stop])


def _dist():
    import torch.distributed as dist
    return dist if dist.is_available() and dist.is_initialized() else None


def max_over_ranks(values, device=None) -> list[float]:
    """Element-wise maximum of a list of floats over all ranks."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    d = _dist()
    if d is not None:
        d.all_reduce(t, op=d.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def sum_over_ranks(values, device=None) -> list[float]:
    """Element-wise sum of a list of floats over all ranks (binary64: counts below 2^53
    stay exact)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    d = _dist()
    if d is not None:
        d.all_reduce(t, op=d.ReduceOp.SUM)
    return [float(v) for v in t.cpu()]


def reduce_rmse(acc):
    """Combine weighted-RMSE accumulators [sum qw e^2, sum qw, sum e^2, max|e|] over ranks.

    ``acc`` is a float64 tensor of 4 entries on this rank's device; a new tensor is
    returned (the input is not modified)."""
    import torch
    sums = acc[:3].clone()
    mx = acc[3:4].clone()
    d = _dist()
    if d is not None:
        d.all_reduce(sums, op=d.ReduceOp.SUM)
        d.all_reduce(mx, op=d.ReduceOp.MAX)
    return torch.cat([sums, mx])


def wrmse(acc) -> float:
    """sqrt(sum qw e^2 / sum qw) of an accumulator."""
    a = [float(v) for v in acc[:2]]
    return (a[0] / a[1]) ** 0.5 if a[1] > 0 else float("nan")


def job_rmse(acc, values, device=None) -> dict:
    """The round-trip statistics of the whole job: every rank passes its accumulator
    [sum qw e^2, sum qw, sum e^2, max|e|] and the number of values it scored; every rank
    gets {wrmse, rmse, maxerr, values} of all ranks together (a collective when a process
    group is initialised: every rank must call it)."""
    total = reduce_rmse(acc)
    n = sum_over_ranks([values], device=device)[0]
    a = [float(v) for v in total]
    return {"wrmse": (a[0] / a[1]) ** 0.5 if a[1] > 0 else float("nan"),
            "rmse": (a[2] / n) ** 0.5 if n > 0 else float("nan"), "maxerr": a[3], "values": int(n)}
