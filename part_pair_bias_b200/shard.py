"""Data-parallel plumbing of the pair-bias path over ranks (one process per GPU).

Jets are independent units of work, so the path shards without any data
exchange: each rank runs whole jets, and the only cross-rank steps are a
barrier around a timed region and a max-reduction of its timings and device
status. Two ways to give ranks their jets:

* weak scaling: every rank draws its own batch of the workload (seed + rank);
* a fixed batch split into contiguous jet ranges of near-equal attention cost
  (sum of m^2, the dominant per-jet term; Particle Transformer pairs scale
  with the square of the multiplicity).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s own batch under weak scaling."""
    return int(seed) + int(rank)


def balanced_ranges(mult: Sequence[int], world: int) -> List[Tuple[int, int]]:
    """Split jets [0, N) into `world` contiguous ranges of near-equal sum of
    m^2. Range r ends at the first jet whose cumulative cost reaches
    (r + 1) / world of the total, so no range exceeds its share by more than
    one jet's cost. Empty ranges are allowed (more ranks than jets)."""
    m = np.asarray(mult, dtype=np.int64)
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = np.cumsum(m * m)
    total = int(cost[-1]) if len(cost) else 0
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        bounds.append(int(np.searchsorted(cost, target, side="left")) + (1 if total else 0))
    bounds.append(len(m))
    bounds = [min(max(b, 0), len(m)) for b in bounds]
    for r in range(1, len(bounds)):           # monotone even when many jets cost 0
        bounds[r] = max(bounds[r], bounds[r - 1])
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def reduce_max(values: Sequence[float], device=None) -> List[float]:
    """Element-wise max over all ranks (identity on a single process)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (the max over ranks)."""
    return float(units_per_rank) * int(world) / float(seconds)
