"""Splitting a batch of independent streams across ranks.

Every (layer, K/V) tensor and every request is a unit with its own codebook
and its own container, so a batch partitions across GPUs with no exchange
step: each rank encodes/decodes its own units with the batched calls, and
the only cross-rank traffic is timing (a barrier and a max-reduce).
"""
from __future__ import annotations

import heapq


def partition(unit_bytes, world: int):
    """Greedy longest-first assignment of units to `world` ranks, balancing
    bytes.  Returns one ascending list of unit indices per rank; every unit
    appears exactly once.  Deterministic for equal inputs."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(unit_bytes)), key=lambda i: (-int(unit_bytes[i]), i))
    heap = [(0, r) for r in range(world)]
    heapq.heapify(heap)
    out = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        out[r].append(i)
        heapq.heappush(heap, (load + int(unit_bytes[i]), r))
    return [sorted(v) for v in out]


def max_over_ranks(value: float, group=None, device=None) -> float:
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
