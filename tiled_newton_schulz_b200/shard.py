"""Data-parallel sharding of a tiled-NS step across ranks (host logic only).

The tiled map has no exchange step: every tile (and so every matrix) is
processed independently ("Hierarchical Muon", abstract: the computation
decomposes into independent small dense matrix operations).  A data-parallel
optimizer can therefore give each rank a subset of the matrices and run one
library call per rank on its subset.  `assign_matrices` balances the subsets by
the NS FLOPs of their tiles (longest-processing-time greedy), keeping each
matrix whole so the CMuon split and the tiling stay inside one call.
"""
from __future__ import annotations

from typing import Sequence


def tile_flops(h: int, w: int, K: int = 5) -> float:
    """Nominal FLOPs of K NS steps on an h x w tile: 2(2a+1)n^3 per step, a = m/n."""
    n, m = min(h, w), max(h, w)
    return K * (4.0 * m * n * n + 2.0 * n ** 3)


def matrix_flops(shape: tuple[int, int], split, T: int, K: int = 5) -> float:
    H, W = shape
    blocks = [(H, W)] if not split else [((H, s) if split[0] == 1 else (s, W)) for s in split[1]]
    total = 0.0
    for h, w in blocks:
        TT = max(h, w) if T <= 0 else T
        for r0 in range(0, h, TT):
            for c0 in range(0, w, TT):
                total += tile_flops(min(TT, h - r0), min(TT, w - c0), K)
    return total


def assign_matrices(shapes: Sequence[tuple[int, int]], splits, T: int, world: int, K: int = 5) -> list[list[int]]:
    """Matrix indices per rank, balanced by NS FLOPs; every index appears once."""
    if world < 1:
        raise ValueError("world must be >= 1")
    splits = splits or [None] * len(shapes)
    cost = [matrix_flops(s, sp, T, K) for s, sp in zip(shapes, splits)]
    order = sorted(range(len(shapes)), key=lambda i: (-cost[i], i))
    load = [0.0] * world
    out: list[list[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        out[r].append(i)
        load[r] += cost[i]
    for lst in out:
        lst.sort()
    return out


def imbalance(shapes, splits, T: int, assignment: list[list[int]], K: int = 5) -> float:
    """max rank load / mean rank load (1.0 = perfect)."""
    splits = splits or [None] * len(shapes)
    loads = [sum(matrix_flops(shapes[i], splits[i], T, K) for i in lst) for lst in assignment]
    mean = sum(loads) / len(loads)
    return max(loads) / mean if mean > 0 else 1.0
