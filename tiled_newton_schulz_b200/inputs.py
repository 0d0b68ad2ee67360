"""Seeded synthetic inputs shared by the tests, the bench and the CPU baseline.

This module draws random matrices and lists workload shapes.  It holds none of
the Newton-Schulz arithmetic and imports neither the library nor the oracle.

Recipes (the pages measure on no public suite; every input is synthetic):

* ``gaussian``: i.i.d. N(0, 1) from numpy's PCG64 ``default_rng(seed)``.
* ``low_rank_plus_noise``: ``U diag(sigma) V^T + noise * N(0, 1)`` with Haar
  U, V (QR of a Gaussian with the column signs fixed by ``sign(diag R)``).
  sigma is ``1/i`` (i = 1..rank) for momentum/gradient matrices and
  ``exp(-i/128)`` for the MoE experts.
* the ``*_torch`` variants draw the same recipe on a torch device with
  ``torch.Generator(device).manual_seed(seed)``; they are used for the large
  7B-shaped set, which is too big to draw on the host.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, Sequence

import numpy as np

# quintic coefficients used for every step by all workloads
QUINTIC = (3.4445, -4.7750, 2.0315)


def gaussian(shape, seed: int, dtype=np.float64) -> np.ndarray:
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


def haar(n: int, k: int, rng: np.random.Generator) -> np.ndarray:
    """n x k matrix with orthonormal columns, Haar distributed."""
    g = rng.standard_normal((n, k))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def sigma_inverse(rank: int) -> np.ndarray:
    return 1.0 / np.arange(1, rank + 1, dtype=np.float64)


def sigma_exp(rank: int, scale: float = 128.0) -> np.ndarray:
    return np.exp(-np.arange(1, rank + 1, dtype=np.float64) / scale)


def low_rank_plus_noise(H: int, W: int, sigma: np.ndarray, noise: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    r = len(sigma)
    U, V = haar(H, r, rng), haar(W, r, rng)
    return (U * sigma[None, :]) @ V.T + noise * rng.standard_normal((H, W))


def signed_permutation(n: int, shift: int, sign_bits: int) -> np.ndarray:
    """n x n signed cyclic permutation: row i has +-1 at column (i + shift) % n.

    The sign of row i is bit (i % 31) of ``sign_bits`` (1 = negative).  Used to
    label tiles so that a misplaced or transposed tile is visible exactly.
    """
    P = np.zeros((n, n))
    for i in range(n):
        P[i, (i + shift) % n] = -1.0 if (sign_bits >> (i % 31)) & 1 else 1.0
    return P


# ---------------------------------------------------------------- torch side

def haar_torch(n: int, k: int, gen, device):
    import torch
    g = torch.randn(n, k, generator=gen, device=device, dtype=torch.float32)
    q, r = torch.linalg.qr(g)
    return q * torch.sign(torch.diagonal(r))[None, :]


def low_rank_plus_noise_torch(H: int, W: int, rank: int, noise: float, seed: int, device,
                              dtype=None, sigma: str = "inverse"):
    """Same recipe as ``low_rank_plus_noise`` drawn on ``device`` (fp32 math)."""
    import torch
    dtype = dtype or torch.bfloat16
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    U, V = haar_torch(H, rank, gen, device), haar_torch(W, rank, gen, device)
    i = torch.arange(1, rank + 1, device=device, dtype=torch.float32)
    s = 1.0 / i if sigma == "inverse" else torch.exp(-i / 128.0)
    out = torch.randn(H, W, generator=gen, device=device, dtype=torch.float32).mul_(noise)
    out.addmm_(U * s[None, :], V.T)
    return out.to(dtype)


def gaussian_torch(H: int, W: int, seed: int, device, dtype=None):
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn(H, W, generator=gen, device=device, dtype=torch.float32).to(dtype or torch.bfloat16)


# ---------------------------------------------------------------- workloads

@dataclass
class MatrixSpec:
    name: str
    rows: int
    cols: int
    split: tuple[int, Sequence[int]] | None = None   # (dim, block sizes) or None


@dataclass
class Workload:
    name: str
    matrices: list[MatrixSpec] = field(default_factory=list)

    @property
    def elements(self) -> int:
        return sum(m.rows * m.cols for m in self.matrices)


def layer_set_2048() -> Workload:
    """One layer set of a d=2048 transformer (Q, K, V, O, MLP up, MLP down)."""
    d = 2048
    return Workload("d2048_layer_set", [
        MatrixSpec("q", d, d), MatrixSpec("k", d, d), MatrixSpec("v", d, d), MatrixSpec("o", d, d),
        MatrixSpec("up", d, 4 * d), MatrixSpec("down", 4 * d, d)])


def llama7b_set(layers: int = 32) -> Workload:
    """All 2-D weights of a Llama-style 7B shape (d=4096, ffn=11008).

    The fused QKV projection (4096 x 12288) is split into three 4096 x 4096
    blocks along its columns (CMuon split) before tiling.
    """
    d, f = 4096, 11008
    mats = []
    for l in range(layers):
        mats += [MatrixSpec(f"l{l}.qkv", d, 3 * d, (1, (d, d, d))), MatrixSpec(f"l{l}.o", d, d),
                 MatrixSpec(f"l{l}.gate", d, f), MatrixSpec(f"l{l}.up", d, f), MatrixSpec(f"l{l}.down", f, d)]
    return Workload(f"llama7b_{layers}l", mats)


def moe_experts(n: int = 64) -> Workload:
    return Workload("moe_experts", [MatrixSpec(f"e{i}", 1024, 4096) for i in range(n)])


def tile_count(rows: int, cols: int, T: int) -> int:
    return math.ceil(rows / T) * math.ceil(cols / T)
