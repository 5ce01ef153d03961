"""Host-side data parallelism for the HSTU hot path.

Users are independent units: attention, KV pages and the block stack are all
per user, so a batch shards across GPUs by user with no collective on the data
path; each GPU keeps its own KV table.  The only cross-rank traffic is timing
and accounting (max of step times, sum of units), done here with
torch.distributed on whatever backend the caller initialised (NCCL on GPUs,
gloo in the CPU tests).
"""

from __future__ import annotations

from typing import List, Sequence

import numpy as np


def attention_cost(lengths: Sequence[int]) -> np.ndarray:
    """Work per user for causal attention: unmasked pairs L (L + 1) / 2."""
    L = np.asarray(lengths, dtype=np.float64)
    return L * (L + 1) / 2


def shard_users(lengths: Sequence[int], world: int) -> List[np.ndarray]:
    """Partition users over `world` ranks, longest-processing-time first.

    Returns, for each rank, the sorted indices of its users.  Every user goes to
    exactly one rank; ties are broken by user index so the result is the same
    on every rank."""
    if world <= 0:
        raise ValueError("world must be positive")
    cost = attention_cost(lengths)
    order = sorted(range(len(cost)), key=lambda u: (-cost[u], u))
    load = [0.0] * world
    parts: List[list] = [[] for _ in range(world)]
    for u in order:
        r = min(range(world), key=lambda k: (load[k], k))
        parts[r].append(u)
        load[r] += cost[u]
    return [np.array(sorted(p), dtype=np.int64) for p in parts]


def contiguous_users(n_users: int, rank: int, world: int) -> np.ndarray:
    """Users [rank * n / world, (rank + 1) * n / world) - the weak-scaling layout
    where every rank owns one per-GPU batch."""
    lo = rank * n_users // world
    hi = (rank + 1) * n_users // world
    return np.arange(lo, hi, dtype=np.int64)


def _reduce(value: float, op: str, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def global_step_time(local_seconds: float, device=None) -> float:
    """Wall time of a data-parallel step: the slowest rank."""
    return _reduce(local_seconds, "max", device)


def global_units(local_units: float, device=None) -> float:
    """Units (FLOPs, candidates) processed by all ranks together."""
    return _reduce(local_units, "sum", device)
