"""Rounding budget of the on-chip arithmetic (CPU, numpy).

The on-chip kernel rounds only the operands of its tensor-core products to 16
bits and accumulates in fp32.  Its operand carries the iterate scaled by
g = sqrt|c/b|, so that S = r(g^2 A) needs no multiply and
    D_P = g^2 A + sign(c/b) S S^T = g^2 (A + (c/b) A^2),
    Bop = r((b/g^2) D_P + a I),   D_X = Bop Xg = g X_{t+1},
and the next operand is r((g_{t+1}/g_t) D_X).  This file re-creates exactly
those rounding points in numpy (round-to-nearest-even bf16 and fp16) and
measures the per-tile relative Frobenius error against the fp64 oracle.  It
shows why the parity tolerance of 3e-2 holds for the step lists the GPU tests
use, and why the sixteen-step GPU case ends in contracting cubic steps:
sixteen quintic steps do not contract and their roundings add up past the
budget.  It shares no code with the library and checks the budget, not the
GPU (the GPU parity tests compare the GPU with the oracle directly).
"""
import numpy as np
import pytest

import oracle
from tiled_newton_schulz_b200 import inputs

BUDGET = 3e-2
QUINTIC = tuple(inputs.QUINTIC)
CUBIC = (1.5, -0.5, 0.0)


def to_bf16(x):
    """Round fp32 values to bf16 (round to nearest, ties to even), as fp64."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def to_fp16(x):
    return np.asarray(x, dtype=np.float16).astype(np.float64)


def to_fp32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def scaled_operand_ns(X, steps, rnd):
    """The on-chip kernel's arithmetic on one square tile (16-bit operands
    by `rnd`, fp32 accumulators)."""
    n = X.shape[0]
    g = [np.sqrt(abs(c / (b if b != 0 else 1.0))) or 1.0 for a, b, c in steps]
    Xo = rnd(g[0] * X / (np.linalg.norm(X) + 1e-7))
    DX = None
    for t, (a, b, c) in enumerate(steps):
        beta = b if b != 0 else 1.0
        DP = to_fp32(Xo @ Xo.T)                                   # g^2 A
        S = rnd(np.sqrt(abs(c / beta)) / g[t] * DP)               # r(g^2 A), or 0 when c = 0
        DP = to_fp32((DP if b != 0 else 0.0) + np.sign(c / beta) * (S @ S.T))
        Bop = rnd((beta / g[t] ** 2) * DP + a * np.eye(n))
        DX = to_fp32(Bop @ Xo)                                    # g X_{t+1}
        if t + 1 < len(steps):
            Xo = rnd((g[t + 1] / g[t]) * DX)
    return DX / g[-1]


def worst_tile_error(steps, T, rnd, seed):
    X = to_bf16(inputs.low_rank_plus_noise(256, 384, inputs.sigma_inverse(32), 0.01, seed=seed))
    c32 = [tuple(float(np.float32(v)) for v in s) for s in steps]
    ref = oracle.ns_tiled(X, T, c32)
    worst = 0.0
    for r0, c0, h, w in oracle.tile_grid(256, 384, T):
        got = scaled_operand_ns(X[r0:r0 + h, c0:c0 + w], steps, rnd)
        want = ref[r0:r0 + h, c0:c0 + w]
        worst = max(worst, np.linalg.norm(got - want) / np.linalg.norm(want))
    return worst


def test_exact_arithmetic_reproduces_the_oracle():
    """With no rounding the scaled-operand algebra is the NS map itself."""
    ident = lambda x: np.asarray(x, dtype=np.float64)
    X = inputs.low_rank_plus_noise(128, 128, inputs.sigma_inverse(32), 0.01, seed=3)
    for steps in ([QUINTIC] * 5, [QUINTIC, CUBIC, (1.5, 0.0, -0.5), (2.0, -1.5, 0.5)]):
        n = X.shape[0]
        g = [np.sqrt(abs(c / (b if b != 0 else 1.0))) or 1.0 for a, b, c in steps]
        Xo = g[0] * X / (np.linalg.norm(X) + 1e-7)
        for t, (a, b, c) in enumerate(steps):
            beta = b if b != 0 else 1.0
            DP = Xo @ Xo.T
            S = ident(np.sqrt(abs(c / beta)) / g[t] * DP)
            DP = (DP if b != 0 else 0.0) + np.sign(c / beta) * (S @ S.T)
            DX = ((beta / g[t] ** 2) * DP + a * np.eye(n)) @ Xo
            if t + 1 < len(steps):
                Xo = (g[t + 1] / g[t]) * DX
        ref = oracle.ns_map(X, steps)
        assert np.linalg.norm(DX / g[-1] - ref) / np.linalg.norm(ref) < 1e-12


@pytest.mark.parametrize("name,steps,T,seed", [
    ("quintic x5", [QUINTIC] * 5, 128, 133),
    ("quintic x5 + cubic x11", [QUINTIC] * 5 + [CUBIC] * 11, 128, 144),
    ("quintic x5 + cubic x11", [QUINTIC] * 5 + [CUBIC] * 11, 64, 80),
    ("mixed", [QUINTIC, CUBIC, (1.5, 0.0, -0.5), (2.0, -1.5, 0.5), QUINTIC, CUBIC], 128, 134),
])
def test_step_lists_of_the_gpu_tests_fit_the_budget(name, steps, T, seed):
    assert worst_tile_error(steps, T, to_bf16, seed) <= BUDGET, name
    assert worst_tile_error(steps, T, to_fp16, seed) <= BUDGET / 3, name


def test_sixteen_quintic_steps_exceed_the_bf16_budget():
    """Sixteen quintic steps do not contract: the bf16 roundings exceed the
    budget by design, not by a kernel fault (fp16 stays near it)."""
    assert worst_tile_error([QUINTIC] * 16, 128, to_bf16, 144) > BUDGET
    assert worst_tile_error([QUINTIC] * 16, 128, to_fp16, 144) < 2 * BUDGET


def _worst_on_tiles(shape, rnd, seeds):
    """Largest per-tile relative Frobenius error and singular-value deviation
    of the emulated kernel arithmetic over Gaussian tiles of `shape` (h <= w)."""
    steps = [QUINTIC] * 5
    c32 = [tuple(float(np.float32(v)) for v in s) for s in steps]
    worst_err = worst_sv = 0.0
    for seed in seeds:
        X = to_bf16(inputs.gaussian(shape, seed=9000 + seed))
        ref = oracle.ns_map(X, c32)
        got = scaled_operand_ns(X, steps, rnd)
        worst_err = max(worst_err, np.linalg.norm(got - ref) / np.linalg.norm(ref))
        sv = np.abs(np.linalg.svd(got, compute_uv=False) - np.linalg.svd(ref, compute_uv=False))
        worst_sv = max(worst_sv, float(sv.max()))
    return worst_err, worst_sv


@pytest.mark.parametrize("shape", [(32, 32), (64, 64), (2, 128), (4, 32), (32, 128)])
def test_thin_tiles_need_more_than_bf16(shape):
    """Tiles with a short side of at most 64: with bf16 operands (8 significant
    bits) their output singular values move past the 0.05 bound (64 x 64
    reaches at least three quarters of it over these seeds and passes it on
    others: no margin for a check over thousands of tiles), with fp16 operands
    (11 bits, the same tensor-core rate) they stay within a third of it.
    This is why a bf16 call rounds such tiles' operands to fp16 on chip (and
    runs them in fp32 when staged)."""
    seeds = range(128)
    err16, sv16 = _worst_on_tiles(shape, to_fp16, seeds)
    assert err16 <= BUDGET / 2 and sv16 <= 0.05 / 3, (err16, sv16)
    errb, svb = _worst_on_tiles(shape, to_bf16, seeds)
    if shape == (64, 64):
        assert svb > 0.75 * 0.05, (errb, svb)
    else:
        assert svb > 0.05 or errb > BUDGET, (errb, svb)


@pytest.mark.parametrize("shape", [(65, 128), (96, 96), (128, 128)])
def test_wider_tiles_fit_the_budget_in_bf16(shape):
    """Tiles with both sides above 64 stay within both bounds with bf16 operands."""
    errb, svb = _worst_on_tiles(shape, to_bf16, range(24))
    assert errb <= BUDGET and svb <= 0.05, (errb, svb)


def test_sixteen_step_list_needs_fp16_on_noisy_tiles():
    """Five quintic then eleven cubic steps multiply a singular value near
    zero by 3.4445^5 x 1.5^11 ~ 4e4: the noise floor of a low-rank-plus-noise
    tile (normalised singular values down to ~1e-5) can end in the steep
    middle of the map, where bf16 operand rounding moves it past the 0.05
    bound and fp16 keeps it within."""
    steps = [QUINTIC] * 5 + [CUBIC] * 11
    c32 = [tuple(float(np.float32(v)) for v in s) for s in steps]
    # the tile of the GPU test's 512 x 768 input whose smallest normalised
    # singular value is 2e-5: the list maps it to 0.74, where the map is steep
    X = to_bf16(inputs.low_rank_plus_noise(512, 768, inputs.sigma_inverse(32), 0.01, seed=19))[256:512, 512:768]
    ref = oracle.ns_map(X, c32)
    dev = {}
    for name, rnd in (("bf16", to_bf16), ("fp16", to_fp16)):
        got = scaled_operand_ns(X, steps, rnd)
        dev[name] = np.abs(np.linalg.svd(got, compute_uv=False) - np.linalg.svd(ref, compute_uv=False)).max()
    assert dev["bf16"] > 0.05 and dev["fp16"] <= 0.05, dev
