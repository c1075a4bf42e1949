"""Assignment of one layer set's matrices to ranks: the multi-GPU split of a full-model solve.

Every matrix of a layer set is an independent dual-scale solve (the DualQuant abstract: one
W ~ diag(r) Q diag(c) fit per weight matrix), so N GPUs share one model by matrix, with no
collective on the data path: each rank solves its share with one dq_solve_batched call and
keeps its results. The split balances the elements per rank (the solve's cost is linear in
them): matrices in decreasing size (ties by index) each go to the rank holding the fewest
elements so far (ties to the lowest rank). This greedy largest-first rule leaves every rank
within one largest matrix of every other.
"""
from __future__ import annotations

from typing import Sequence


def assign(sizes: Sequence[int], world: int) -> list:
    """Per-rank lists of matrix indices (ascending) for matrices of the given element counts."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if any(int(s) < 0 for s in sizes):
        raise ValueError("sizes must be non-negative")
    load = [0] * world
    parts = [[] for _ in range(world)]
    order = sorted(range(len(sizes)), key=lambda i: (-int(sizes[i]), i))
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        parts[r].append(i)
        load[r] += int(sizes[i])
    return [sorted(p) for p in parts]


def loads(sizes: Sequence[int], parts: Sequence[Sequence[int]]) -> list:
    """Elements per rank of an assignment."""
    return [sum(int(sizes[i]) for i in p) for p in parts]
