"""Layer sharding across ranks (one process per GPU).

Layers are independent units of the merge path, so a model's layers are
split across ranks with no collective on the data path: greedy longest-
processing-time assignment by element count, deterministic on every rank.
"""
from __future__ import annotations

from typing import Sequence


def shard_layers(numels: Sequence[int], world: int) -> list[list[int]]:
    """Indices of the layers each rank owns. Every layer is owned exactly once;
    layers are taken largest first and given to the least-loaded rank (ties to
    the lower rank), then each rank's list is sorted back into model order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(numels)), key=lambda k: (-int(numels[k]), k))
    load = [0] * world
    owned: list[list[int]] = [[] for _ in range(world)]
    for k in order:
        r = min(range(world), key=lambda q: (load[q], q))
        owned[r].append(k)
        load[r] += int(numels[k])
    return [sorted(o) for o in owned]


def imbalance(numels: Sequence[int], shards: Sequence[Sequence[int]]) -> float:
    """max rank load / mean rank load (1.0 = perfectly balanced)."""
    loads = [sum(int(numels[k]) for k in s) for s in shards]
    mean = sum(loads) / len(loads)
    return max(loads) / mean if mean else 1.0
