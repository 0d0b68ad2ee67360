"""The on-chip and the staged path on the same calls (HIMUON_FORCE_PATH=staged
sends a T = 128 call through the staged GEMMs), and resuming a Muon step from
saved state.  Needs a B200."""
import io

import numpy as np
import pytest

import oracle
from tests.parity_util import bf16_ulp, per_tile_errors, to_np
from tiled_newton_schulz_b200 import inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

QUINTIC = inputs.QUINTIC
C32 = [tuple(float(np.float32(v)) for v in QUINTIC)] * 5
TOL16 = 3e-2


@pytest.fixture(scope="module")
def hm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_newton_schulz_b200 import himuon
    himuon.load()
    return himuon


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda", torch.bfloat16)


@pytest.mark.parametrize("T", [128, 256])
def test_forced_staged_path_agrees_with_on_chip(hm, monkeypatch, T):
    """The on-chip kernels (T = 128: one CTA per tile group; T = 256: a CTA
    pair per tile) and the staged GEMMs on the same call."""
    X = inputs.low_rank_plus_noise(384, 512, inputs.sigma_inverse(16), 0.01, seed=21)
    x = dev(X)
    p = hm.params(T, QUINTIC, steps=5)
    y_chip = torch.empty_like(x)
    hm.ns_tiled([x], [y_chip], p)
    n0 = hm.launch_count()
    monkeypatch.setenv("HIMUON_FORCE_PATH", "staged")
    y_stg = torch.empty_like(x)
    hm.ns_tiled([x], [y_stg], p)
    torch.cuda.synchronize()
    assert hm.launch_count() - n0 > 1          # pack, GEMMs, normalise, unpack: not the one on-chip launch
    monkeypatch.delenv("HIMUON_FORCE_PATH")
    assert hm.device_status() == 0
    ref = oracle.ns_tiled(to_np(x), T, C32)
    a, b = to_np(y_chip), to_np(y_stg)
    assert per_tile_errors(a, ref, T).max() <= TOL16
    assert per_tile_errors(b, ref, T).max() <= TOL16
    assert per_tile_errors(a, b, T).max() <= TOL16


@pytest.mark.parametrize("T", [128, 256])
def test_forced_staged_momentum_step_same_momentum(hm, monkeypatch, T):
    """Both paths form M' = mu M + G in fp32 and store it rounded to nearest
    bf16: bit-identical.  W' agrees within the update's tolerance."""
    H, W = 256, 384
    w0 = 0.02 * inputs.gaussian((H, W), seed=1)
    m0 = inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=2)
    g0 = inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=3)
    p = hm.params(T, QUINTIC, steps=5)
    out = {}
    for path in ("chip", "staged"):
        if path == "staged":
            monkeypatch.setenv("HIMUON_FORCE_PATH", "staged")
        w, m, g = dev(w0), dev(m0), dev(g0)
        hm.momentum_step([w], [m], [g], 0.95, 0.02, p)
        assert hm.device_status() == 0
        out[path] = (to_np(w), to_np(m))
    monkeypatch.delenv("HIMUON_FORCE_PATH")
    assert np.array_equal(out["chip"][1], out["staged"][1])
    W2, _, O = oracle.momentum_step(to_np(dev(w0)), to_np(dev(m0)), to_np(dev(g0)), 0.95, 0.02, T, C32)
    bound = np.linalg.norm(0.5 * bf16_ulp(W2)) + float(np.float32(0.02)) * TOL16 * np.linalg.norm(O)
    for path in out:
        assert np.linalg.norm(out[path][0] - W2) <= bound


def test_resume_from_saved_state_is_bit_identical(hm):
    """Two steps in place, or one step, save W and M, load them into fresh
    tensors and take the second step: the same bits (the library keeps no
    state between calls but cached plans)."""
    H, W = 384, 512
    w0 = 0.02 * inputs.gaussian((H, W), seed=4)
    m0 = inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=5)
    g1 = dev(inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=6))
    g2 = dev(inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=7))
    p = hm.params(128, QUINTIC, steps=5)
    w, m = dev(w0), dev(m0)
    hm.momentum_step([w], [m], [g1], 0.95, 0.02, p)
    buf = io.BytesIO()
    torch.save({"W": w.cpu(), "M": m.cpu()}, buf)
    hm.momentum_step([w], [m], [g2], 0.95, 0.02, p)
    buf.seek(0)
    st = torch.load(buf)
    w_r, m_r = st["W"].to("cuda"), st["M"].to("cuda")
    hm.momentum_step([w_r], [m_r], [g2], 0.95, 0.02, p)
    assert hm.device_status() == 0
    assert torch.equal(w, w_r) and torch.equal(m, m_r)


def partial_signed_permutation(H, W, k, seed):
    """H x W (H <= W) with one +-1 per row, in column (k i + 5) mod W: distinct
    columns when gcd(k, W) = 1, so X X^T = I and every singular value is 1."""
    assert np.gcd(k, W) == 1 and H <= W
    P = np.zeros((H, W))
    P[np.arange(H), (np.arange(H) * k + 5) % W] = np.random.default_rng(seed).choice([-1.0, 1.0], H)
    return P


@pytest.mark.parametrize("H,W", [(4608, 4608), (4224, 8320)])
def test_full_ns_of_permutation_beyond_one_band_of_row_tiles(hm, H, W):
    """Full NS where the staged GEMMs have more than 32 row tiles (36 and 33:
    a full band of 32 and a partial one in the grouped CTA order).  X is a
    signed (partial) permutation, so every product is exact up to the operand
    rounding and NS(X) = phi(1/sqrt(H)) X: the output's support and signs must
    equal X's exactly, every magnitude must be the same, and that magnitude is
    the oracle's map of a 2 x 2 matrix with the same normalised singular value
    (diag(1, sqrt(H - 1)) has Frobenius norm sqrt(H)).  A GEMM tile written to
    the wrong place, or not written, breaks the support."""
    X = partial_signed_permutation(H, W, 7, seed=H)
    x = dev(X)
    y = torch.empty_like(x)
    hm.ns_full([x], [y], hm.params(0, QUINTIC, steps=5))
    assert hm.device_status() == 0
    Y = to_np(y)
    nz = X != 0
    assert np.array_equal(Y != 0, nz)
    assert np.array_equal(np.sign(Y[nz]), np.sign(X[nz]))
    mags = np.abs(Y[nz])
    assert np.all(mags == mags[0])
    want = oracle.ns_map(np.diag([1.0, np.sqrt(H - 1.0)]), C32)[0, 0]
    assert abs(mags[0] - want) <= TOL16 * want
