"""Per-matrix tile sizes in one call (a runtime tile-size schedule, the
"Hierarchical Muon" abstract) on the GPU.

The library groups a call's matrices by their T and runs each group as a call
with that single T.  So every matrix of a mixed call must come out bit for bit
as the single-T call gives it, and match the fp64 oracle at its own T
(tolerances as in test_gpu_parity.py: per-tile relative Frobenius error
<= 3e-2 in bf16, M' within one bf16 ulp).  The cost measurement and the
budgeted choice run through the library as well.
"""
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
MU, LR = 0.95, 0.02

# on chip (T = 64 packed, T = 128 with a ragged edge), staged (256, 512) and full NS
SHAPES = [(256, 384), (384, 640), (640, 832), (300, 500), (512, 512), (200, 1000), (512, 768)]
TILES = [64, 128, 256, 0, 512, 128, 256]


@pytest.fixture(scope="module")
def hm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_newton_schulz_b200 import himuon
    himuon.load()
    return himuon


def state(seed):
    dev = torch.device("cuda", 0)
    W = [(inputs.gaussian_torch(h, w, seed + 3 * i, dev, torch.float32) * 0.02).to(torch.bfloat16)
         for i, (h, w) in enumerate(SHAPES)]
    M = [inputs.low_rank_plus_noise_torch(h, w, 16, 0.01, seed + 3 * i + 1, dev) for i, (h, w) in enumerate(SHAPES)]
    G = [inputs.low_rank_plus_noise_torch(h, w, 16, 0.01, seed + 3 * i + 2, dev) for i, (h, w) in enumerate(SHAPES)]
    return W, M, G


def clone(xs):
    return [x.clone() for x in xs]


def test_mixed_tiles_momentum_step_equals_single_tile_calls_and_oracle(hm):
    W, M, G = state(100)
    W0, M0, G0 = [to_np(x) for x in W], [to_np(x) for x in M], [to_np(x) for x in G]
    W2, M2, G2 = clone(W), clone(M), clone(G)
    O, O2 = [torch.empty_like(x) for x in M], [torch.empty_like(x) for x in M]
    hm.momentum_step(W, M, G, MU, LR, hm.params(128, QUINTIC, steps=5, tiles=TILES), update_out=O)
    for T in sorted(set(TILES)):
        idx = [i for i, t in enumerate(TILES) if t == T]
        hm.momentum_step([W2[i] for i in idx], [M2[i] for i in idx], [G2[i] for i in idx], MU, LR,
                         hm.params(T, QUINTIC, steps=5), update_out=[O2[i] for i in idx])
    assert hm.device_status() == 0
    for i, T in enumerate(TILES):
        assert torch.equal(O[i], O2[i]), (i, T)
        assert torch.equal(W[i], W2[i]) and torch.equal(M[i], M2[i]), (i, T)
        To = T if T > 0 else max(SHAPES[i])     # the oracle takes the whole matrix as one T x T tile
        Wr, Mr, Or = oracle.momentum_step(W0[i], M0[i], G0[i], MU, LR, To, C32)
        assert np.all(np.abs(to_np(M[i]) - Mr) <= bf16_ulp(Mr)), (i, T)
        assert per_tile_errors(to_np(O[i]), Or, T).max() <= TOL16, (i, T)


def test_mixed_tiles_ns_with_split_and_gram(hm):
    """Standard NS and Gram NS (fp16, restart at t = 3) with T = 256 on a
    split fused tensor, T = 128 and the whole matrix in one call each."""
    shapes = [(512, 1536), (384, 640), (640, 256)]
    X = [torch.from_numpy(inputs.low_rank_plus_noise(h, w, inputs.sigma_exp(min(h, w), 32.0), 1e-3, 11 + i))
         .to(device="cuda", dtype=torch.bfloat16) for i, (h, w) in enumerate(shapes)]
    splits = [(1, (512, 512, 512)), None, None]
    tiles = [256, 128, 0]
    pg = dict(compute=hm.FP16, restart=(3,))
    Y, Yg = [torch.empty_like(x) for x in X], [torch.empty_like(x) for x in X]
    hm.ns_tiled(X, Y, hm.params(0, QUINTIC, steps=5, tiles=tiles), splits=splits)
    hm.gram_ns(X, Yg, hm.params(0, QUINTIC, steps=5, tiles=tiles, **pg), splits=splits)
    assert hm.device_status() == 0
    for i, T in enumerate(tiles):
        Ys, Ygs = torch.empty_like(X[i]), torch.empty_like(X[i])
        hm.ns_tiled([X[i]], [Ys], hm.params(T, QUINTIC, steps=5), splits=[splits[i]])
        hm.gram_ns([X[i]], [Ygs], hm.params(T, QUINTIC, steps=5, **pg), splits=[splits[i]])
        assert hm.device_status() == 0
        assert torch.equal(Y[i], Ys) and torch.equal(Yg[i], Ygs), (i, T)
        x = to_np(X[i])
        blocks = [slice(512 * j, 512 * (j + 1)) for j in range(3)] if splits[i] else [slice(None)]
        for sl in blocks:
            xb = x[:, sl]
            ref = oracle.ns_tiled(xb, T if T > 0 else max(xb.shape), C32)
            refg = oracle.gram_ns_tiled(xb, T, C32, restart=(3,))
            assert per_tile_errors(to_np(Y[i])[:, sl], ref, T).max() <= TOL16, (i, T)
            assert per_tile_errors(to_np(Yg[i])[:, sl], refg, T).max() <= TOL16, (i, T)


def test_measured_costs_and_budgeted_choice(hm):
    from tiled_newton_schulz_b200 import schedule
    shapes = [(1024, 1024), (1024, 2752), (2752, 1024), (1024, 1024)]
    costs = schedule.measure_costs(shapes, candidates=(64, 128, 256, 512, 0), reps=2, min_elements=1 << 22)
    assert len(costs) == 4 and costs[0] == costs[3]
    step_costs = schedule.measure_costs(shapes, candidates=(128, 0), reps=2, min_elements=1 << 22, op="step")
    assert all(set(c) == {128, 0} and all(v > 0 for v in c.values()) for c in step_costs)
    for c in costs:
        assert set(c) == {64, 128, 256, 512, 0}
        assert all(np.isfinite(v) and v > 0 for v in c.values())
    cheapest = schedule.choose_tiles(costs, 0.0)
    widest = schedule.choose_tiles(costs, float("inf"))
    assert all(schedule.quality(a) >= schedule.quality(b) for a, b in zip(widest, cheapest))
    budget = 0.5 * (schedule.modeled_cost(costs, cheapest) + schedule.modeled_cost(costs, widest))
    mid = schedule.choose_tiles(costs, budget)
    assert schedule.modeled_cost(costs, mid) <= budget
    # the chosen mix runs in one call
    dev = torch.device("cuda", 0)
    X = [inputs.gaussian_torch(h, w, 30 + i, dev) for i, (h, w) in enumerate(shapes)]
    Y = [torch.empty_like(x) for x in X]
    hm.ns_tiled(X, Y, hm.params(0, QUINTIC, steps=5, tiles=mid))
    assert hm.device_status() == 0
    assert all(torch.isfinite(y.float()).all() for y in Y)
