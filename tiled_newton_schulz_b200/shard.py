"""Data-parallel sharding of a tiled-NS Muon step across ranks (host logic).

The tiled map has no exchange step: every tile (and so every matrix) is
processed independently ("Hierarchical Muon", abstract: the computation
decomposes into independent small dense matrix operations).  A data-parallel
optimizer can therefore give each rank a subset of the matrices and run one
library call per rank on its subset.  `assign_matrices` balances the subsets by
the NS FLOPs of their tiles (longest-processing-time greedy), keeping each
matrix whole so the CMuon split and the tiling stay inside one call.
`sharded_momentum_step` is the step around it: gradients summed onto each
matrix's owner, the owner's library call, the new weights broadcast back.
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


def owners(assignment: list[list[int]], n: int) -> list[int]:
    """Rank that owns each of the n matrices; every index must appear once."""
    own = [-1] * n
    for r, lst in enumerate(assignment):
        for i in lst:
            if not 0 <= i < n or own[i] != -1:
                raise ValueError(f"matrix {i} is out of range or assigned twice")
            own[i] = r
    if -1 in own:
        raise ValueError(f"matrix {own.index(-1)} is not assigned")
    return own


def sharded_momentum_step(W, M, G, mu: float, lr: float, params, assignment: list[list[int]], splits=None,
                          average: bool = True, group=None, step_fn=None) -> None:
    """One data-parallel Muon step with the optimizer work sharded by matrix.

    Every rank holds the replicated weights W and its local gradients G for
    all n matrices; the momentum M[i] lives only on the rank that owns matrix i
    (`assignment`, e.g. from ``assign_matrices``; other ranks may pass None).

    1. G[i] is summed onto its owner (``dist.reduce``) and, with `average`,
       divided there by the world size.
    2. Each rank runs the tiled-NS Muon step (M <- mu M + G; W <- W - lr NS(M))
       on its own matrices in one call: ``step_fn(W_own, M_own, G_own, mu, lr,
       p, splits=...)``, by default ``himuon.momentum_step``.  `params` is the
       himuon params, or a callable that maps the owned indices to them (for a
       per-matrix tile list).
    3. The owner broadcasts the updated W[i] to every rank.

    Tiles are independent, so there is no other exchange.  All ranks issue the
    same collectives in matrix order; before the first one they agree (an
    all-reduce of a flag) that every rank's inputs are complete, and raise
    together otherwise, so that no rank is left waiting in a collective.
    """
    import torch
    import torch.distributed as dist

    n = len(W)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    own = owners(assignment, n)
    if len(assignment) != world:
        raise ValueError("assignment has one list per rank")
    mine = [i for i in range(n) if own[i] == rank]
    problem = ""
    if len(G) != n or len(M) != n:
        problem = "W, M and G need one entry per matrix"
    elif any(M[i] is None for i in mine):
        problem = f"rank {rank} owns a matrix without momentum"
    elif any(W[i] is None or G[i] is None or W[i].shape != G[i].shape for i in range(n)):
        problem = "W and G need matching tensors for every matrix"
    flag = torch.tensor([0 if problem else 1], dtype=torch.int32,
                        device=W[0].device if dist.get_backend(group) == "nccl" else "cpu")
    dist.all_reduce(flag, op=dist.ReduceOp.MIN, group=group)
    if problem:
        raise ValueError(problem)
    if int(flag.item()) == 0:
        raise ValueError("another rank's inputs to the sharded step are incomplete")

    global_rank = [dist.get_global_rank(group, r) for r in range(world)] if group is not None else list(range(world))
    works = [dist.reduce(G[i], dst=global_rank[own[i]], op=dist.ReduceOp.SUM, group=group, async_op=True)
             for i in range(n)]
    for w in works:
        w.wait()
    if mine:
        if average and world > 1:
            for i in mine:
                G[i].div_(world)
        if step_fn is None:
            from . import himuon
            step_fn = himuon.momentum_step
        p = params(mine) if callable(params) else params
        step_fn([W[i] for i in mine], [M[i] for i in mine], [G[i] for i in mine], mu, lr, p,
                splits=None if splits is None else [splits[i] for i in mine])
    works = [dist.broadcast(W[i], src=global_rank[own[i]], group=group, async_op=True) for i in range(n)]
    for w in works:
        w.wait()
