"""Pins of the fp64 oracle to facts other than its own code (CPU only).

Each check comes from the mathematics the pages state, not from re-typing the
oracle's loops:

* "Gram Newton-Schulz" page, sec. 3 (mathematical interpretation): the NS
  iterate keeps the singular vectors of the normalised input and applies the
  step polynomials p_t(x) = a_t x + b_t x^3 + c_t x^5 to its singular values,
  so NS(X) = U phi(S / (||X||_F + eps)) V^T with phi = p_K o ... o p_1.  The
  test computes this with numpy's SVD.
* same page, sec. 2/5: Gram NS is mathematically equivalent to standard NS;
  sec. 6: the restart changes nothing in exact arithmetic.
* "Hierarchical Muon" abstract: every tile's output is the NS map of that tile
  alone, placed back where the tile came from.
* CMuon article: each functional block of a fused tensor is orthogonalised on
  its own.

The per-step coefficient lists below are deliberately all different so that a
reversed step order, a swapped coefficient or a dropped term changes the
result.
"""
import numpy as np
import pytest

import oracle
from tiled_newton_schulz_b200 import inputs

EPS = 1e-7
CFG = [inputs.QUINTIC]
C5 = [(3.4445, -4.7750, 2.0315), (2.9, -3.1, 1.1), (2.2, -1.6, 0.45), (1.9, -1.3, 0.4), (1.6, -0.8, 0.2)]


def phi(x, coeffs):
    x = np.asarray(x, dtype=np.float64)
    for a, b, c in coeffs:
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def ns_by_svd(X, coeffs, eps=EPS, safety=1.0):
    """The SVD route: U phi(sigma / (safety (||X||_F + eps))) V^T."""
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    nrm = np.sqrt(np.sum(X * X))
    return (U * phi(s / ((nrm + eps) * safety), coeffs)[None, :]) @ Vt


def rel(a, b):
    d = np.linalg.norm(a - b)
    n = np.linalg.norm(b)
    return d / n if n > 0 else d


SHAPES = [(1, 1), (1, 7), (7, 1), (2, 2), (3, 5), (5, 3), (6, 6), (6, 9), (9, 6), (16, 24), (24, 16)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("coeffs", [CFG * 5, C5], ids=["quintic", "per_step"])
def test_ns_map_equals_svd_closed_form(shape, coeffs):
    X = inputs.gaussian(shape, seed=hash(shape) % 1000)
    out = oracle.ns_map(X, coeffs)
    assert rel(out, ns_by_svd(X, coeffs)) < 1e-11


def test_step_order_is_visible():
    X = inputs.gaussian((8, 12), seed=5)
    fwd = oracle.ns_map(X, C5)
    rev = oracle.ns_map(X, C5[::-1])
    assert rel(fwd, ns_by_svd(X, C5)) < 1e-11
    assert rel(rev, fwd) > 1e-3          # the order of the steps matters


def test_eps_sits_beside_the_norm():
    # With ||X||_F ~ 1e-6 the +eps in the denominator moves the singular values
    # by ~10%; the closed form with eps matches, the one without does not.
    X = inputs.gaussian((5, 8), seed=11)
    X = X / np.linalg.norm(X) * 1e-6
    out = oracle.ns_map(X, CFG * 5)
    assert rel(out, ns_by_svd(X, CFG * 5)) < 1e-11
    assert rel(out, ns_by_svd(X, CFG * 5, eps=0.0)) > 1e-3


@pytest.mark.parametrize("shape", [(3, 5), (6, 6), (9, 4)])
@pytest.mark.parametrize("safety", [1.05, 2.0])
def test_safety_factor_divides_the_normalised_input(shape, safety):
    """"Gram Newton-Schulz" page, sec. 6 implementation notes: the input is
    divided by the safety factor (1.05 in the example) after normalisation, so
    the singular values entering phi are sigma / (safety (||X||_F + eps))."""
    X = inputs.gaussian(shape, seed=shape[0] + 17 * shape[1])
    for co in (C5, C5[:2]):
        out = oracle.ns_map(X, co, safety=safety)
        assert rel(out, ns_by_svd(X, co, safety=safety)) < 1e-11
        g = oracle.gram_ns(X, co, restart=(2,), safety=safety)
        assert rel(g, ns_by_svd(X, co, safety=safety)) < 1e-10
        t = oracle.ns_tiled(X, 2, co, safety=safety)
        for r0, c0, h, w in oracle.tile_grid(*shape, 2):
            blk = X[r0:r0 + h, c0:c0 + w]
            assert rel(t[r0:r0 + h, c0:c0 + w], ns_by_svd(blk, co, safety=safety)) < 1e-11
    # two steps leave the factor visible (five converged steps nearly hide it)
    out = oracle.ns_map(X, C5[:2], safety=safety)
    assert rel(out, ns_by_svd(X, C5[:2])) > 1e-3                       # the factor is applied
    assert rel(out, ns_by_svd(X, C5[:2], safety=1.0 / safety)) > 1e-3  # ... as a divisor


def test_safety_factor_scales_norm_plus_eps():
    # ||X||_F ~ 1e-6: dividing (||X||_F + eps) by the factor and dividing
    # ||X||_F alone before adding eps give visibly different results.
    X = inputs.gaussian((4, 7), seed=12)
    X = X / np.linalg.norm(X) * 1e-6
    out = oracle.ns_map(X, CFG * 5, safety=2.0)
    assert rel(out, ns_by_svd(X, CFG * 5, safety=2.0)) < 1e-11
    U, sv, Vt = np.linalg.svd(X, full_matrices=False)
    other = (U * phi(sv / (2.0 * np.linalg.norm(X) + EPS), CFG * 5)[None, :]) @ Vt
    assert rel(out, other) > 1e-3


@pytest.mark.parametrize("x", [2.5, -0.3, 1e-9, -7.0])
def test_scalar_closed_form(x):
    out = oracle.ns_map(np.array([[x]]), C5)
    want = np.sign(x) * phi(abs(x) / (abs(x) + EPS), C5)
    assert abs(out[0, 0] - want) <= 1e-13 * max(1.0, abs(want))


def test_one_step_at_unit_input_is_a_plus_b_plus_c():
    # p(1) = a + b + c = 0.701 for the quintic coefficients (up to the eps shift)
    out = oracle.ns_map(np.array([[1.0]]), CFG, K=1)
    a, b, c = inputs.QUINTIC
    assert abs(out[0, 0] - (a + b + c)) < 1e-5
    assert abs((a + b + c) - 0.701) < 1e-12


@pytest.mark.parametrize("n", [1, 5, 33])
def test_vector_closed_form(n):
    v = inputs.gaussian((n,), seed=n)
    nv = np.linalg.norm(v)
    want = phi(nv / (nv + EPS), C5) * v / nv
    assert rel(oracle.ns_map(v[None, :], C5)[0], want) < 1e-12
    assert rel(oracle.ns_map(v[:, None], C5)[:, 0], want) < 1e-12


@pytest.mark.parametrize("n", [3, 8, 17])
def test_scaled_signed_permutation(n):
    c = 0.37
    P = inputs.signed_permutation(n, shift=2, sign_bits=0b1011001)
    out = oracle.ns_map(c * P, C5)
    want = phi(c / (c * np.sqrt(n) + EPS), C5) * P
    assert np.max(np.abs(out - want)) < 1e-13


def test_zero_tile_gives_zero():
    out = oracle.ns_tiled(np.zeros((6, 10)), 4, CFG, K=5)
    assert np.all(out == 0.0) and np.all(np.isfinite(out))


@pytest.mark.parametrize("H,W,T", [(8, 12, 4), (10, 7, 4), (9, 13, 5), (6, 6, 16), (12, 5, 8), (5, 12, 8), (7, 7, 7)])
def test_tiled_each_tile_is_ns_of_that_tile(H, W, T):
    X = inputs.gaussian((H, W), seed=H * 100 + W * 10 + T)
    out = oracle.ns_tiled(X, T, C5)
    count = 0
    for r0 in range(0, H, T):
        for c0 in range(0, W, T):
            blk = X[r0:r0 + T, c0:c0 + T]
            assert rel(out[r0:r0 + T, c0:c0 + T], ns_by_svd(blk, C5)) < 1e-11
            count += 1
    assert count == -(-H // T) * -(-W // T)


def test_tiled_with_large_T_is_full_ns():
    X = inputs.gaussian((12, 20), seed=3)
    assert rel(oracle.ns_tiled(X, 20, C5), ns_by_svd(X, C5)) < 1e-11
    assert rel(oracle.ns_tiled(X, 4096, C5), ns_by_svd(X, C5)) < 1e-11
    # a smaller T is a different (local) map, not an approximation of it
    assert rel(oracle.ns_tiled(X, 4, C5), ns_by_svd(X, C5)) > 1e-2


@pytest.mark.parametrize("H,W,T", [(12, 12, 4), (11, 14, 4), (16, 9, 8)])
def test_tiled_integer_coded_reassembly(H, W, T):
    """Tile t holds c_t times a signed (partial) permutation with its own shift
    and signs; the output must keep every support position and sign exactly,
    so a misplaced, swapped or transposed tile shows up."""
    X = np.zeros((H, W))
    for t, (r0, c0, h, w) in enumerate(oracle.tile_grid(H, W, T)):
        P = inputs.signed_permutation(T, shift=t % T, sign_bits=(t * 2654435761) & 0x7FFFFFFF)
        X[r0:r0 + h, c0:c0 + w] = (0.5 + 0.1 * t) * P[:h, :w]
    out = oracle.ns_tiled(X, T, C5)
    assert np.array_equal(np.sign(out), np.sign(X))
    for (r0, c0, h, w) in oracle.tile_grid(H, W, T):
        blk, ob = X[r0:r0 + h, c0:c0 + w], out[r0:r0 + h, c0:c0 + w]
        k = np.count_nonzero(blk)
        if k:
            c = np.max(np.abs(blk))
            want = phi(c / (c * np.sqrt(k) + EPS), C5)
            assert np.allclose(np.abs(ob[blk != 0]), want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("shape", [(6, 10), (10, 6), (16, 16), (5, 40), (1, 9)])
@pytest.mark.parametrize("restart", [(), (3,), (2, 4), (2, 3), (1,), (1, 2, 3, 4, 5), (9,)])
def test_gram_ns_equals_standard_ns(shape, restart):
    X = inputs.gaussian(shape, seed=shape[0] * 7 + shape[1])
    g = oracle.gram_ns(X, C5, restart=restart)
    assert rel(g, ns_by_svd(X, C5)) < 1e-10
    assert rel(g, oracle.ns_map(X, C5)) < 1e-10


def test_gram_ns_on_low_rank_spectrum():
    X = inputs.low_rank_plus_noise(24, 96, inputs.sigma_exp(24, 8.0), 1e-3, seed=4)
    assert rel(oracle.gram_ns(X, CFG * 5, restart=(3,)), ns_by_svd(X, CFG * 5)) < 1e-10


@pytest.mark.parametrize("T", [8, 16, 40])
def test_gram_ns_tiled_is_tilewise_svd_map(T):
    """Tiled Gram NS: each tile (ragged edges included, tall ones too) is
    mapped by the SVD closed form of its own NS polynomial, independently of
    its neighbours: a tile scaled by 1000 changes no other tile."""
    X = inputs.gaussian((50, 70), seed=T)
    g = oracle.gram_ns_tiled(X, T, C5, restart=(3,))
    for r0, c0, h, w in oracle.tile_grid(50, 70, T):
        assert rel(g[r0:r0 + h, c0:c0 + w], ns_by_svd(X[r0:r0 + h, c0:c0 + w], C5)) < 1e-10
    Y = X.copy()
    Y[:T, :T] *= 1000.0
    gy = oracle.gram_ns_tiled(Y, T, C5, restart=(3,))
    assert np.array_equal(gy[T:, :], g[T:, :]) and np.array_equal(gy[:T, T:], g[:T, T:])
    assert rel(gy[:T, :T], g[:T, :T]) < 1e-7           # scale-invariant up to the eps in the norm
    assert rel(oracle.gram_ns_tiled(X, 0, C5), oracle.gram_ns(X, C5)) == 0.0


def test_momentum_step_closed_form():
    rng = np.random.default_rng(9)
    W, M, G = (rng.standard_normal((6, 9)) for _ in range(3))
    mu, eta = 0.95, 0.02
    W2, M2, O = oracle.momentum_step(W, M, G, mu, eta, T=64, coeffs=C5)
    mu32, eta32 = float(np.float32(mu)), float(np.float32(eta))
    assert np.array_equal(M2, mu32 * M + G)
    assert rel(O, ns_by_svd(mu32 * M + G, C5)) < 1e-11
    assert rel(W2, W - eta32 * ns_by_svd(mu32 * M + G, C5)) < 1e-13


def test_split_blocks_are_independent():
    X = inputs.gaussian((8, 24), seed=21)
    split = (1, (8, 8, 8))
    out = oracle.ns_tiled_split(X, 4096, C5, split=split)
    for j in range(3):
        blk = X[:, 8 * j:8 * (j + 1)]
        assert rel(out[:, 8 * j:8 * (j + 1)], ns_by_svd(blk, C5)) < 1e-11
    assert rel(out, ns_by_svd(X, C5)) > 1e-2   # splitting changes full-matrix NS
    # with T dividing the block size, the split does not change tiled NS
    assert np.array_equal(oracle.ns_tiled_split(X, 4, C5, split=split), oracle.ns_tiled(X, 4, C5))


def test_split_rows_and_ragged_blocks():
    X = inputs.gaussian((10, 6), seed=22)
    split = (0, (3, 7))
    out = oracle.ns_tiled_split(X, 4, C5, split=split)
    assert rel(out[:3], oracle.ns_tiled(X[:3], 4, C5)) == 0.0
    assert rel(out[3:], oracle.ns_tiled(X[3:], 4, C5)) == 0.0
    for (r0, c0, h, w) in oracle.tile_grid(7, 6, 4):
        blk = X[3 + r0:3 + r0 + h, c0:c0 + w]
        assert rel(out[3 + r0:3 + r0 + h, c0:c0 + w], ns_by_svd(blk, C5)) < 1e-11


def test_split_validation():
    with pytest.raises(ValueError):
        oracle.split_blocks((8, 24), (1, (8, 8)))
    with pytest.raises(ValueError):
        oracle.split_blocks((8, 24), (1, (8, 0, 16)))


def test_tile_grid_indexing():
    tiles = list(oracle.tile_grid(10, 7, 4))
    assert tiles == [(0, 0, 4, 4), (0, 4, 4, 3), (4, 0, 4, 4), (4, 4, 4, 3), (8, 0, 2, 4), (8, 4, 2, 3)]
