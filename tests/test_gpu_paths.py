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


def test_forced_staged_path_agrees_with_on_chip(hm, monkeypatch):
    X = inputs.low_rank_plus_noise(384, 512, inputs.sigma_inverse(16), 0.01, seed=21)
    x = dev(X)
    p = hm.params(128, QUINTIC, steps=5)
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
    ref = oracle.ns_tiled(to_np(x), 128, C32)
    a, b = to_np(y_chip), to_np(y_stg)
    assert per_tile_errors(a, ref, 128).max() <= TOL16
    assert per_tile_errors(b, ref, 128).max() <= TOL16
    assert per_tile_errors(a, b, 128).max() <= TOL16


def test_forced_staged_momentum_step_same_momentum(hm, monkeypatch):
    """Both paths form M' = mu M + G in fp32 and store it rounded to nearest
    bf16: bit-identical.  W' agrees within the update's tolerance."""
    H, W = 256, 384
    w0 = 0.02 * inputs.gaussian((H, W), seed=1)
    m0 = inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=2)
    g0 = inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=3)
    p = hm.params(128, QUINTIC, steps=5)
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
    W2, _, O = oracle.momentum_step(to_np(dev(w0)), to_np(dev(m0)), to_np(dev(g0)), 0.95, 0.02, 128, C32)
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
