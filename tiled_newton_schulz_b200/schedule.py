"""Runtime tile-size schedules for tiled NS (host logic).

"Hierarchical Muon: Tiled Newton-Schulz Updates for Efficient Muon
Optimization" (abstract) names runtime tile-size schedules among the things
the tiled map allows: T is a parameter of the same per-tile map, so it can
change from one optimizer step to the next and differ between matrices.  The
pages give no rule for choosing T.  This module supplies the pieces a trainer
needs, and the library runs their result in one call
(``himuon.params(..., tiles=[T per matrix])``):

* ``TileSchedule``: T as a piecewise-constant function of the optimizer step,
  with overrides for single matrices.
* ``choose_tiles``: per matrix, the largest tile a time budget allows, from a
  table of measured costs.  Larger tiles keep more of the coupling between
  rows and columns that tiling discards (the abstract: spectral interactions
  survive inside a tile and are dropped across tile boundaries); the whole
  matrix (T <= 0, full-matrix NS) is the limit.
* ``measure_costs``: that table, timed with CUDA events through the library
  on the device, for the distinct shapes of a matrix set.
"""
from __future__ import annotations

import math
import numbers
from typing import Mapping, Sequence


def quality(T: int) -> float:
    """Order of tile sizes by how much of the matrix one tile couples:
    larger is closer to full-matrix NS, and T <= 0 (the whole matrix) is the
    top."""
    return math.inf if T <= 0 else float(T)


class TileSchedule:
    """Tile size by optimizer step and matrix.

    default     T for every matrix before the first milestone.
    milestones  [(first_step, T), ...]: from optimizer step `first_step` on
                (0-based), T replaces the default; later milestones win.
    per_matrix  {matrix index: T, or a milestone list of its own} overriding
                the schedule for that matrix.
    """

    def __init__(self, default: int = 128, milestones: Sequence[tuple[int, int]] = (),
                 per_matrix: Mapping[int, int | Sequence[tuple[int, int]]] | None = None):
        self.default = int(default)
        self.milestones = self._check(milestones)
        self.per_matrix = {}
        for i, v in (per_matrix or {}).items():
            self.per_matrix[int(i)] = int(v) if isinstance(v, numbers.Integral) else self._check(v)

    @staticmethod
    def _check(ms):
        out = sorted((int(s), int(t)) for s, t in ms)
        if any(s < 0 for s, _ in out):
            raise ValueError("milestone steps start at 0")
        if len({s for s, _ in out}) != len(out):
            raise ValueError("two milestones at the same step")
        return out

    @staticmethod
    def _at(step: int, base: int, ms) -> int:
        T = base
        for s, t in ms:
            if step >= s:
                T = t
            else:
                break
        return T

    def tile_at(self, step: int, matrix: int | None = None) -> int:
        T = self._at(step, self.default, self.milestones)
        if matrix is not None and matrix in self.per_matrix:
            v = self.per_matrix[matrix]
            T = v if isinstance(v, int) else self._at(step, T, v)
        return T

    def tiles(self, step: int, n: int) -> list[int]:
        """One T per matrix of an n-matrix call at this optimizer step."""
        return [self.tile_at(step, i) for i in range(n)]


def pareto_chain(cost: Mapping[int, float]) -> list[tuple[int, float]]:
    """The candidates of one matrix that no other beats on both counts
    (cheaper or as cheap, and at least as large a tile), by increasing cost
    and tile size."""
    items = sorted(cost.items(), key=lambda kv: (kv[1], -quality(kv[0])))
    chain, best = [], -math.inf
    for T, t in items:
        if not math.isfinite(t) or t < 0:
            raise ValueError(f"cost of T={T} is {t}")
        if quality(T) > best:
            chain.append((int(T), float(t)))
            best = quality(T)
    return chain


def choose_tiles(costs: Sequence[Mapping[int, float]], budget: float) -> list[int]:
    """One T per matrix: the largest tiles whose summed cost stays within
    `budget` (same unit as the costs).

    costs[i] maps each candidate T of matrix i to its cost (T <= 0: the whole
    matrix).  Every matrix starts at its cheapest candidate; then, greedily,
    the cheapest single upgrade to the next larger tile on that matrix's
    Pareto chain is taken while the total fits.  When even the cheapest choice
    exceeds the budget, the cheapest choice is returned.
    """
    if not costs:
        return []
    chains = [pareto_chain(c) for c in costs]
    if any(not ch for ch in chains):
        raise ValueError("a matrix has no candidate tile size")
    pos = [0] * len(chains)
    total = sum(ch[0][1] for ch in chains)
    while True:
        pick = None
        for i, ch in enumerate(chains):
            if pos[i] + 1 < len(ch):
                d = ch[pos[i] + 1][1] - ch[pos[i]][1]
                if total + d <= budget and (pick is None or d < pick[0]):
                    pick = (d, i)
        if pick is None:
            break
        total += pick[0]
        pos[pick[1]] += 1
    return [ch[p][0] for ch, p in zip(chains, pos)]


def modeled_cost(costs: Sequence[Mapping[int, float]], tiles: Sequence[int]) -> float:
    """Sum of the per-matrix costs of a tile choice."""
    return float(sum(c[int(T)] for c, T in zip(costs, tiles)))


def measure_costs(shapes: Sequence[tuple[int, int]], splits=None, candidates: Sequence[int] = (128, 256, 512, 0),
                  coeffs=None, steps: int = 5, compute: int | None = None, reps: int = 3,
                  min_elements: int = 1 << 27, device=None, op: str = "ns") -> list[dict[int, float]]:
    """Seconds per matrix at each candidate T, measured on the device.

    op = "ns" times ``ns_tiled`` (in -> out); op = "step" times the whole Muon
    step ``momentum_step`` (W, M, G; M and W updated in place), which is what a
    trainer's budget covers.  Matrices with the same shape and split share one
    measurement: up to ceil(min_elements / elements) of them (at most as many
    as the set has) run as one batched call on Gaussian inputs, timed with
    CUDA events over `reps` calls after one untimed call, and the time is
    divided by the count.  Returns costs[i][T] for every matrix i of
    `shapes`, ready for ``choose_tiles``.
    """
    import torch
    from . import himuon as hm
    from .inputs import QUINTIC, gaussian_torch

    if op not in ("ns", "step"):
        raise ValueError(f"op must be 'ns' or 'step', not {op!r}")
    hm.load()
    coeffs = QUINTIC if coeffs is None else coeffs
    compute = hm.BF16 if compute is None else compute
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    splits = [None] * len(shapes) if splits is None else list(splits)
    keys = {}
    for i, (shape, sp) in enumerate(zip(shapes, splits)):
        key = (tuple(int(v) for v in shape), None if sp is None else (int(sp[0]), tuple(int(v) for v in sp[1])))
        keys.setdefault(key, []).append(i)
    dtype = torch.float32 if compute == hm.FP32 else (torch.float16 if compute == hm.FP16 else torch.bfloat16)
    stream = torch.cuda.current_stream(dev)
    out = [dict() for _ in shapes]
    for k, ((H, W), sp) in enumerate(keys):
        members = keys[((H, W), sp)]
        count = min(len(members), max(1, -(-min_elements // (H * W))))
        X = [gaussian_torch(H, W, 7000 + 97 * k + j, dev, torch.float32).to(dtype) for j in range(count)]
        if op == "ns":
            Y = [torch.empty_like(x) for x in X]     # O
        else:
            Y = [gaussian_torch(H, W, 9000 + 97 * k + j, dev, torch.float32).to(dtype) for j in range(count)]  # G
        Wt = [(0.02 * gaussian_torch(H, W, 8000 + 97 * k + j, dev, torch.float32)).to(dtype)
              for j in range(count)] if op == "step" else None
        spl = None if sp is None else [(sp[0], list(sp[1]))] * count
        for T in candidates:
            p = hm.params(int(T), coeffs, steps=steps, compute=compute)
            code = hm.OP_MOMENTUM_STEP if op == "step" else (hm.OP_NS_TILED if T > 0 else hm.OP_NS_FULL)
            need = hm.workspace_size(X, p, code, spl)
            ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev) if need else None

            def call():
                if op == "step":
                    hm.momentum_step(Wt, X, Y, 0.95, 0.02, p, splits=spl, workspace=ws, stream=stream)
                else:
                    hm.ns_tiled(X, Y, p, splits=spl, workspace=ws, stream=stream)

            call()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                call()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            sec = e0.elapsed_time(e1) / 1e3 / reps / count
            for i in members:
                out[i][int(T)] = sec
            del ws
        del X, Y, Wt
    st = hm.device_status()
    if st != 0:
        raise hm.HimuonError(st, "measure_costs")
    return out
