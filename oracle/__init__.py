"""fp64 CPU oracle for the tiled Newton-Schulz map (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
may import this package.  The library path never does, and this package never
imports the library: the two share no code.

The arithmetic lives in ``himuon_oracle.c`` (plain fp64 loops, optionally
OpenMP over independent tiles).  This module only builds that file, converts
inputs to float64 and walks the split/tile structure:

* ``ns_map``       -- Algorithm 1 of the "Gram Newton-Schulz" page (sec. 3).
* ``ns_tiled``     -- the HiMuon tiling ("Hierarchical Muon", abstract).
* ``gram_ns``      -- Gram NS of the "Gram Newton-Schulz" page (sec. 5-6): the
  same map computed through the Gram matrix, with restarts.
* ``split_blocks`` -- the CMuon split of a fused tensor into its functional
  blocks (CMuon article).
* ``momentum_step`` -- the Muon recap update (sec. 3):
  ``M' = mu M + G``, ``W' = W - eta * NS(M')``.

Each is pinned in ``tests/test_oracle_pins.py`` to things other than itself:
the SVD closed form of the NS iterate (sec. 3, "mathematical interpretation"),
scalar closed forms, exact equality of Gram NS and standard NS (sec. 2 and 5),
and brute-force index checks of the tiling.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Iterable, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "himuon_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

EPS = 1e-7  # "epsilon = 1e-7", Gram Newton-Schulz page, Algorithm 1


def build(force: bool = False) -> str:
    """Compile himuon_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        i64, ci = ctypes.c_int64, ctypes.c_int
        cd = ctypes.c_double
        lib.oracle_ns_map.argtypes = [dp, i64, i64, i64, ci, dp, cd, cd, dp, i64]
        lib.oracle_ns_map.restype = ci
        lib.oracle_ns_tiled.argtypes = [dp, i64, i64, i64, i64, ci, dp, cd, cd, dp, i64]
        lib.oracle_ns_tiled.restype = ci
        lib.oracle_gram_ns.argtypes = [dp, i64, i64, i64, ci, dp, cd, cd,
                                       ctypes.POINTER(ctypes.c_int), ci, dp, i64]
        lib.oracle_gram_ns.restype = ci
        lib.oracle_num_threads.restype = ci
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a (CPU/GPU) torch tensor."""
    if hasattr(x, "detach"):  # torch tensor: go through float64 on the host
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _coeffs(coeffs, K: int | None = None) -> tuple[np.ndarray, int]:
    c = np.asarray(coeffs, dtype=np.float64).reshape(-1, 3)
    if K is not None and c.shape[0] == 1 and K > 1:
        c = np.repeat(c, K, axis=0)
    return np.ascontiguousarray(c), c.shape[0]


def ns_map(x, coeffs, K: int | None = None, eps: float = EPS, safety: float = 1.0) -> np.ndarray:
    """Standard NS (Algorithm 1) of one matrix, in fp64.  ``safety`` divides the
    normalised input (sec. 6 implementation notes; 1.0 = off)."""
    X = _f64(x)
    c, K = _coeffs(coeffs, K)
    h, w = X.shape
    out = np.zeros((h, w), dtype=np.float64)
    rc = _load().oracle_ns_map(_ptr(X), w, h, w, K, _ptr(c), eps, float(safety), _ptr(out), w)
    if rc != 0:
        raise MemoryError("oracle_ns_map failed")
    return out


def ns_tiled(x, T: int, coeffs, K: int | None = None, eps: float = EPS, safety: float = 1.0) -> np.ndarray:
    """HiMuon: NS applied to each T x T tile (ragged edges smaller), in place."""
    X = _f64(x)
    c, K = _coeffs(coeffs, K)
    H, W = X.shape
    out = np.zeros((H, W), dtype=np.float64)
    rc = _load().oracle_ns_tiled(_ptr(X), W, H, W, int(T), K, _ptr(c), eps, float(safety), _ptr(out), W)
    if rc != 0:
        raise RuntimeError(f"oracle_ns_tiled failed ({rc})")
    return out


def gram_ns(x, coeffs, K: int | None = None, restart: Sequence[int] = (3,), eps: float = EPS,
            safety: float = 1.0) -> np.ndarray:
    """Gram NS of one matrix (sec. 5-6): R = X X^T, Q = I, per step P = p_t(R),
    Q <- P Q, R <- P R P; output Q X.  ``restart`` lists the 1-based steps
    before which X <- Q X, R <- X X^T, Q <- I."""
    X = _f64(x)
    c, K = _coeffs(coeffs, K)
    h, w = X.shape
    out = np.zeros((h, w), dtype=np.float64)
    rs = (ctypes.c_int * max(1, len(restart)))(*restart)
    rc = _load().oracle_gram_ns(_ptr(X), w, h, w, K, _ptr(c), eps, float(safety), rs, len(restart), _ptr(out), w)
    if rc != 0:
        raise MemoryError("oracle_gram_ns failed")
    return out


def gram_ns_tiled(x, T: int, coeffs, K: int | None = None, restart: Sequence[int] = (3,),
                  eps: float = EPS, safety: float = 1.0) -> np.ndarray:
    """Gram NS applied to each T x T tile ("Hierarchical Muon" abstract: the
    same map per tile, reassembled; ragged edge tiles smaller).  T <= 0 or at
    least the matrix's sides: the whole matrix."""
    X = _f64(x)
    H, W = X.shape
    if T <= 0 or T >= max(H, W):
        return gram_ns(X, coeffs, K, restart, eps, safety)
    out = np.zeros((H, W), dtype=np.float64)
    for r0, c0, h, w in tile_grid(H, W, T):
        out[r0:r0 + h, c0:c0 + w] = gram_ns(X[r0:r0 + h, c0:c0 + w], coeffs, K, restart, eps, safety)
    return out


def split_blocks(shape: tuple[int, int], split: tuple[int, Sequence[int]] | None):
    """CMuon split: list of (row0, col0, rows, cols) blocks of a fused matrix.

    ``split = (dim, sizes)`` cuts dimension ``dim`` (0 = rows, 1 = columns)
    into consecutive blocks of the given sizes, which must sum to that
    dimension.  ``None`` keeps the matrix whole.
    """
    H, W = shape
    if split is None:
        return [(0, 0, H, W)]
    dim, sizes = split
    total = H if dim == 0 else W
    if sum(sizes) != total or any(s <= 0 for s in sizes):
        raise ValueError("split sizes must be positive and sum to the split dimension")
    blocks, off = [], 0
    for s in sizes:
        blocks.append((off, 0, s, W) if dim == 0 else (0, off, H, s))
        off += s
    return blocks


def ns_tiled_split(x, T: int, coeffs, K: int | None = None, split=None, eps: float = EPS,
                   safety: float = 1.0) -> np.ndarray:
    """Split (CMuon) then tile (HiMuon) each block; blocks are independent."""
    X = _f64(x)
    out = np.zeros_like(X)
    for (r0, c0, h, w) in split_blocks(X.shape, split):
        out[r0:r0 + h, c0:c0 + w] = ns_tiled(X[r0:r0 + h, c0:c0 + w], T, coeffs, K, eps, safety)
    return out


def momentum(M, G, mu: float) -> np.ndarray:
    """Muon recap: M' = mu M + G (mu as the fp32 value the library receives)."""
    mu = float(np.float32(mu))
    return mu * _f64(M) + _f64(G)


def momentum_step(W, M, G, mu: float, eta: float, T: int, coeffs, K: int | None = None,
                  split=None, eps: float = EPS, safety: float = 1.0):
    """One Muon step with tiled NS: returns (W', M', O) in fp64."""
    Mp = momentum(M, G, mu)
    O = ns_tiled_split(Mp, T, coeffs, K, split, eps, safety)
    eta = float(np.float32(eta))
    return _f64(W) - eta * O, Mp, O


def tile_grid(H: int, W: int, T: int) -> Iterable[tuple[int, int, int, int]]:
    """(row0, col0, h, w) of every tile, row-major from the top-left corner."""
    for r0 in range(0, H, T):
        for c0 in range(0, W, T):
            yield r0, c0, min(T, H - r0), min(T, W - c0)
