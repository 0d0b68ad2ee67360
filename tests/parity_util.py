"""Comparison helpers for the GPU parity tests (CPU side, numpy fp64).

Metrics (tolerances are stated in the tests that use them):
* per-tile relative Frobenius error ||Y - Y*||_F / ||Y*||_F (absolute error
  for an all-zero reference tile);
* sorted singular values of a tile (or whole matrix) within an absolute bound;
* bit-exact support/sign patterns for integer-coded tiles.
"""
import numpy as np


def tiles(H, W, T):
    T = max(H, W) if T <= 0 else T
    for r0 in range(0, H, T):
        for c0 in range(0, W, T):
            yield r0, c0, min(T, H - r0), min(T, W - c0)


def per_tile_errors(Y, Yref, T):
    H, W = Yref.shape
    out = []
    for r0, c0, h, w in tiles(H, W, T):
        a, b = Y[r0:r0 + h, c0:c0 + w], Yref[r0:r0 + h, c0:c0 + w]
        nb = np.linalg.norm(b)
        d = np.linalg.norm(a - b)
        out.append(d / nb if nb > 0 else d)
    return np.array(out)


def max_sv_diff(Y, Yref, T, sample=None, seed=0):
    """Largest |sorted sv(Y_tile) - sorted sv(Yref_tile)| over (a sample of) tiles."""
    H, W = Yref.shape
    tl = list(tiles(H, W, T))
    if sample is not None and len(tl) > sample:
        idx = np.random.default_rng(seed).choice(len(tl), sample, replace=False)
        tl = [tl[i] for i in idx]
    worst = 0.0
    for r0, c0, h, w in tl:
        sa = np.linalg.svd(Y[r0:r0 + h, c0:c0 + w], compute_uv=False)
        sb = np.linalg.svd(Yref[r0:r0 + h, c0:c0 + w], compute_uv=False)
        worst = max(worst, float(np.max(np.abs(sa - sb))))
    return worst


def bf16_ulp(x):
    """Spacing of bfloat16 numbers at |x| (x as float64 array)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 7), 2.0 ** -133)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)
