"""Partition a weight set's tensors over ranks (one process per GPU).

The decode needs no exchange step: tensors are independent, so each rank
decodes its own share from its own HBM. The share is balanced by the bytes a
decode moves (container read + BF16 written), by longest-processing-time
assignment: tensors in decreasing size, each to the rank with the least load so
far (ties to the lower rank). Every tensor goes to exactly one rank, and no
rank's load exceeds another's by more than the largest tensor's.
"""
from __future__ import annotations


def partition(loads: list[int], world: int) -> list[list[int]]:
    """Indices of `loads` for each of `world` ranks (each list ascending)."""
    if world < 1:
        raise ValueError("world must be at least 1")
    order = sorted(range(len(loads)), key=lambda i: (-int(loads[i]), i))
    total = [0] * world
    parts: list[list[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (total[k], k))
        parts[r].append(i)
        total[r] += int(loads[i])
    return [sorted(p) for p in parts]


def rank_loads(loads: list[int], parts: list[list[int]]) -> list[int]:
    return [sum(int(loads[i]) for i in p) for p in parts]
