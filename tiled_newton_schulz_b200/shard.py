"""Data-parallel sharding of a tiled-NS Muon step across ranks (host logic).

The tiled map has no exchange step: every tile (and so every matrix) is
processed independently ("Hierarchical Muon", abstract: the computation
decomposes into independent small dense matrix operations).  A data-parallel
optimizer can therefore give each rank a subset of the matrices and run one
library call per rank on its subset.  `assign_matrices` balances the subsets by
the NS FLOPs of their tiles (longest-processing-time greedy), keeping each
matrix whole so the CMuon split and the tiling stay inside one call.

Two steps are built on it:

* `FlatShards` + `flat_sharded_step`: the weights and the gradients of all
  matrices live in one flat buffer each, laid out so that every (bucket, rank)
  pair owns one contiguous, equally sized slot.  A step is a reduce-scatter of
  the gradients (each rank receives the averaged gradients of its own
  matrices, bucket by bucket), the rank's fused library step on its own
  matrices (the momentum lives only there), and an in-place all-gather of the
  weights.  Matrices are views of the flat buffers: no packing copies.  Buckets
  let one bucket's collectives overlap another bucket's step.
* `sharded_momentum_step`: the same step with one reduce and one broadcast per
  matrix, for matrices that cannot share a flat buffer.
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


# ---------------------------------------------------------------- flat buffers

_ALIGN = 128   # elements: every matrix and slot starts 256-byte aligned (16-bit storage)


def _round(x: int, m: int = _ALIGN) -> int:
    return (x + m - 1) // m * m


class FlatShards:
    """Placement of n matrices in one flat buffer for a sharded step.

    Each matrix is owned by one rank (`assign_matrices`, balanced by NS FLOPs)
    and belongs to one of `buckets` buckets of that rank (consecutive owned
    matrices, split evenly by elements).  The buffer is bucket-major:

        [bucket 0: slot(rank 0) | slot(rank 1) | ... ][bucket 1: ...] ...

    and every slot of bucket b has the same size, `slot_elems[b]` (the largest
    rank's share, padded), so a bucket is one contiguous world x slot region:
    exactly the layout `reduce_scatter_tensor` and `all_gather_into_tensor`
    take.  Matrix i is the row-major (rows x cols) view at `offset[i]`.
    `mine_offset[i]` is its offset inside its rank's own slots laid end to end
    (the layout of a per-rank buffer such as the momentum).
    """

    def __init__(self, shapes, splits, T, world: int, buckets: int = 1, K: int = 5, tiles=None):
        n = len(shapes)
        self.shapes = [tuple(int(v) for v in s) for s in shapes]
        self.world = int(world)
        self.splits = list(splits) if splits is not None else [None] * n
        if tiles is None:
            self.assignment = assign_matrices(self.shapes, self.splits, T, world, K)
        else:
            self.assignment = _assign_per_tile(self.shapes, self.splits, tiles, world, K)
        self.owner = owners(self.assignment, n)
        nb = max(1, int(buckets))
        elems = [_round(h * w) for h, w in self.shapes]
        # per rank: its matrices in order, cut into nb consecutive groups of ~equal elements
        self.bucket_of = [0] * n
        per = [[[] for _ in range(nb)] for _ in range(world)]
        for r, lst in enumerate(self.assignment):
            total = sum(elems[i] for i in lst)
            acc = 0
            for i in lst:
                b = min(nb - 1, int(acc * nb / total)) if total else 0
                per[r][b].append(i)
                self.bucket_of[i] = b
                acc += elems[i]
        self.members = per                     # members[rank][bucket] = matrix indices
        self.slot_elems = [_round(max(sum(elems[i] for i in per[r][b]) for r in range(world)) or _ALIGN)
                           for b in range(nb)]
        self.bucket_base = []
        base = 0
        for b in range(nb):
            self.bucket_base.append(base)
            base += world * self.slot_elems[b]
        self.total = base
        self.offset = [0] * n
        self.mine_offset = [0] * n
        for r in range(world):
            mine = 0
            for b in range(nb):
                off = self.bucket_base[b] + r * self.slot_elems[b]
                for i in per[r][b]:
                    self.offset[i] = off
                    self.mine_offset[i] = mine + (off - self.bucket_base[b] - r * self.slot_elems[b])
                    off += elems[i]
                mine += self.slot_elems[b]
        self.mine_total = sum(self.slot_elems)
        self.buckets = nb

    def views(self, flat):
        """Matrix views (rows x cols) of a flat buffer laid out by this placement."""
        return [flat[o:o + h * w].view(h, w) for o, (h, w) in zip(self.offset, self.shapes)]

    def mine_views(self, flat_mine, rank: int):
        """Views of this rank's own matrices in a per-rank buffer of mine_total
        elements (None for the matrices it does not own)."""
        out = [None] * len(self.shapes)
        for i, (h, w) in enumerate(self.shapes):
            if self.owner[i] == rank:
                o = self.mine_offset[i]
                out[i] = flat_mine[o:o + h * w].view(h, w)
        return out

    def bucket(self, flat, b: int):
        return flat[self.bucket_base[b]:self.bucket_base[b] + self.world * self.slot_elems[b]]

    def slot(self, flat, b: int, rank: int):
        o = self.bucket_base[b] + rank * self.slot_elems[b]
        return flat[o:o + self.slot_elems[b]]

    def imbalance(self, T, K: int = 5) -> float:
        return imbalance(self.shapes, self.splits, T, self.assignment, K)


def _assign_per_tile(shapes, splits, tiles, world, K):
    """LPT assignment with a tile size per matrix."""
    cost = [matrix_flops(s, sp, t, K) for s, sp, t in zip(shapes, splits, tiles)]
    order = sorted(range(len(shapes)), key=lambda i: (-cost[i], i))
    load = [0.0] * world
    out = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        out[r].append(i)
        load[r] += cost[i]
    for lst in out:
        lst.sort()
    return out


def flat_sharded_step(W_flat, G_flat, M_mine, shards: FlatShards, mu: float, lr: float, params, average: bool = True,
                      group=None, step_fn=None, stream=None, O_flat=None) -> None:
    """One data-parallel Muon step over matrices laid out by `shards`.

    W_flat: the replicated weights (same values on every rank), G_flat: this
    rank's local gradients, both flat buffers of shards.total elements laid
    out by `shards`; M_mine: this rank's momentum, a flat buffer of
    shards.mine_total elements (`shards.mine_views`).  Per bucket b:

    1. reduce-scatter of bucket b of G_flat, in place: this rank's slot now
       holds the gradients of its own matrices summed (averaged with
       `average`) over the ranks;
    2. ``step_fn(W_own, M_own, G_own, mu, lr, p, splits=...)`` (by default
       ``himuon.momentum_step``) on this rank's matrices of bucket b: M <- mu M
       + G, W <- W - lr NS(M), in place in the flat buffers;
    3. all-gather of bucket b of W_flat, in place: every rank gets the new
       weights of every matrix.

    The reduce-scatters are all issued first, so bucket b + 1's runs under
    bucket b's step, and bucket b's all-gather under bucket b + 1's step.
    Every rank issues the same collectives in the same order.  `params` is the
    himuon params or a callable of the owned indices (per-matrix tile lists).
    On NCCL the collectives follow the current CUDA stream (or `stream`).
    `O_flat` (optional, laid out like W_flat) receives the update NS(M) of this
    rank's own matrices (step_fn's update_out).
    """
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nccl = dist.get_backend(group) == "nccl"
    problem = ""
    if world != shards.world:
        problem = f"placement made for {shards.world} ranks, group has {world}"
    elif W_flat.numel() != shards.total or G_flat.numel() != shards.total or M_mine.numel() != shards.mine_total:
        problem = f"rank {rank}: flat buffers do not match the placement"
    # every rank learns whether all inputs are in order before the first
    # collective, so that none is left waiting in one
    flag = torch.tensor([0 if problem else 1], dtype=torch.int32, device=W_flat.device if nccl else "cpu")
    dist.all_reduce(flag, op=dist.ReduceOp.MIN, group=group)
    if problem:
        raise ValueError(problem)
    if int(flag.item()) == 0:
        raise ValueError("another rank's inputs to the sharded step are incomplete")
    op = dist.ReduceOp.AVG if (nccl and average) else dist.ReduceOp.SUM
    if step_fn is None:
        from . import himuon
        step_fn = himuon.momentum_step
    Wv, Gv, Mv = shards.views(W_flat), shards.views(G_flat), shards.mine_views(M_mine, rank)
    Ov = shards.views(O_flat) if O_flat is not None else None
    ctx = torch.cuda.stream(stream) if (stream is not None and nccl) else _nullcontext()
    with ctx:
        rs = []
        for b in range(shards.buckets):
            bucket = shards.bucket(G_flat, b)
            rs.append(dist.reduce_scatter_tensor(shards.slot(G_flat, b, rank), bucket, op=op, group=group,
                                                 async_op=True) if world > 1 else None)
        ag = []
        for b in range(shards.buckets):
            if rs[b] is not None:
                rs[b].wait()
            mine = shards.members[rank][b]
            if mine:
                if average and world > 1 and not nccl:
                    for i in mine:
                        Gv[i].div_(world)
                p = params(mine) if callable(params) else params
                kw = {"splits": [shards.splits[i] for i in mine]}
                if stream is not None and nccl:
                    kw["stream"] = stream
                if Ov is not None:
                    kw["update_out"] = [Ov[i] for i in mine]
                step_fn([Wv[i] for i in mine], [Mv[i] for i in mine], [Gv[i] for i in mine], mu, lr, p, **kw)
            if world > 1:
                ag.append(dist.all_gather_into_tensor(shards.bucket(W_flat, b), shards.slot(W_flat, b, rank),
                                                      group=group, async_op=True))
        for w in ag:
            w.wait()


class _nullcontext:
    def __enter__(self):
        return None

    def __exit__(self, *exc):
        return False
