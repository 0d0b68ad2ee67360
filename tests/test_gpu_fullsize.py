"""Full-size parity (needs a B200 and ~60 GB of device memory).

Each workload runs at its real size in the launch configuration the bench
uses; the fp64 oracle then recomputes a seeded sample of tiles (or whole
experts) from the inputs the GPU saw, and the GPU outputs at those places are
compared element by element.  Tolerances as in test_gpu_parity.py: per-tile
relative Frobenius error <= 3e-2 and singular values within 0.05 (bf16, tiles
of short side >= 64); M' within one bf16 ulp.
"""
import numpy as np
import pytest

import oracle
from tests.parity_util import bf16_ulp
from tiled_newton_schulz_b200 import inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

QUINTIC = inputs.QUINTIC
C32 = [tuple(float(np.float32(v)) for v in QUINTIC)] * 5
TOL16, SVTOL = 3e-2, 0.05


@pytest.fixture(scope="module")
def hm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_newton_schulz_b200 import himuon
    himuon.load()
    return himuon


def rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def svd_dev(a, b):
    return np.max(np.abs(np.linalg.svd(a, compute_uv=False) - np.linalg.svd(b, compute_uv=False)))


def f64(t):
    return t.detach().double().cpu().numpy()


def sample_tiles(mats, T, n, seed):
    """(matrix index, block origin col/row, tile row0, col0, h, w) of n seeded tiles."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        i = int(rng.integers(len(mats)))
        (H, W), split = mats[i]
        if split:
            j = int(rng.integers(len(split[1])))
            off = sum(split[1][:j])
            bh, bw = (H, split[1][j]) if split[0] == 1 else (split[1][j], W)
            br, bc = (0, off) if split[0] == 1 else (off, 0)
        else:
            bh, bw, br, bc = H, W, 0, 0
        tr = int(rng.integers(-(-bh // T)))
        tc = int(rng.integers(-(-bw // T)))
        r0, c0 = br + tr * T, bc + tc * T
        out.append((i, r0, c0, min(T, br + bh - r0), min(T, bc + bw - c0)))
    return out


@pytest.mark.parametrize("T", [128, 256])
def test_llama7b_full_step_sampled_tiles(hm, T):
    """The 7B-shaped set (32 layers, QKV split), one Muon step as the bench
    runs it: T = 128 on chip, T = 256 staged in chunks of at most 16 GB."""
    import bench
    dev = torch.device("cuda", 0)
    mats, W, M, G = bench.make_state(dev, seed_base=0)
    splits = [s for _, s in mats]
    picks = sample_tiles(mats, T, 24, seed=T)
    before = [(f64(W[i][r:r + h, c:c + w]), f64(M[i][r:r + h, c:c + w]), f64(G[i][r:r + h, c:c + w]))
              for (i, r, c, h, w) in picks]
    p = hm.params(T, QUINTIC, steps=5, chunk_bytes=16 << 30)
    ws = hm.workspace_size(M, p, hm.OP_MOMENTUM_STEP, splits)
    wsb = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev) if ws else None
    hm.momentum_step(W, M, G, bench.MU, bench.LR, p, splits=splits, workspace=wsb)
    assert hm.device_status() == 0
    lr32 = float(np.float32(bench.LR))
    for (i, r, c, h, w), (w0, m0, g0) in zip(picks, before):
        W2, M2, O = oracle.momentum_step(w0, m0, g0, bench.MU, bench.LR, T, C32)
        mg, wg = f64(M[i][r:r + h, c:c + w]), f64(W[i][r:r + h, c:c + w])
        assert np.all(np.abs(mg - M2) <= bf16_ulp(M2))
        # the update the GPU applied, recovered from W (bf16 rounding of W' bounded)
        bound = np.linalg.norm(0.5 * bf16_ulp(W2)) + lr32 * TOL16 * np.linalg.norm(O)
        assert np.linalg.norm(wg - W2) <= bound
    del W, M, G, wsb
    torch.cuda.empty_cache()


def test_llama7b_update_out_sampled_tiles(hm):
    """Same set, T = 128, asking for O itself on a 4-layer slice (memory)."""
    import bench
    dev = torch.device("cuda", 0)
    mats, W, M, G = bench.make_state(dev, seed_base=7, layers=4)
    splits = [s for _, s in mats]
    O = [torch.empty_like(x) for x in M]
    picks = sample_tiles(mats, 128, 32, seed=5)
    before = [(f64(M[i][r:r + h, c:c + w]), f64(G[i][r:r + h, c:c + w])) for (i, r, c, h, w) in picks]
    hm.momentum_step(None, M, G, bench.MU, bench.LR, hm.params(128, QUINTIC, steps=5), splits=splits,
                     update_out=O)
    assert hm.device_status() == 0
    for (i, r, c, h, w), (m0, g0) in zip(picks, before):
        ref = oracle.ns_map(oracle.momentum(m0, g0, bench.MU), C32)
        got = f64(O[i][r:r + h, c:c + w])
        assert rel(got, ref) <= TOL16
        assert svd_dev(got, ref) <= SVTOL


def test_d2048_layer_set_sampled_tiles(hm):
    dev = torch.device("cuda", 0)
    wl = inputs.layer_set_2048()
    M = [inputs.low_rank_plus_noise_torch(m.rows, m.cols, 64, 0.01, 10 + i, dev) for i, m in enumerate(wl.matrices)]
    G = [inputs.low_rank_plus_noise_torch(m.rows, m.cols, 64, 0.01, 20 + i, dev) for i, m in enumerate(wl.matrices)]
    O = [torch.empty_like(x) for x in M]
    mats = [((m.rows, m.cols), None) for m in wl.matrices]
    picks = sample_tiles(mats, 128, 48, seed=2)
    before = [(f64(M[i][r:r + h, c:c + w]), f64(G[i][r:r + h, c:c + w])) for (i, r, c, h, w) in picks]
    hm.momentum_step(None, M, G, 0.95, 0.02, hm.params(128, QUINTIC, steps=5), update_out=O)
    assert hm.device_status() == 0
    for (i, r, c, h, w), (m0, g0) in zip(picks, before):
        mp = oracle.momentum(m0, g0, 0.95)
        assert np.all(np.abs(f64(M[i][r:r + h, c:c + w]) - mp) <= bf16_ulp(mp))
        ref = oracle.ns_map(mp, C32)
        got = f64(O[i][r:r + h, c:c + w])
        assert rel(got, ref) <= TOL16 and svd_dev(got, ref) <= SVTOL


@pytest.mark.parametrize("T", [32, 64, 128, 256, 512])
def test_4096x16384_sweep_sampled_tiles(hm, T):
    dev = torch.device("cuda", 0)
    X = inputs.gaussian_torch(4096, 16384, 3, dev)
    Y = torch.empty_like(X)
    p = hm.params(T, QUINTIC, steps=5)
    hm.ns_tiled([X], [Y], p)
    assert hm.device_status() == 0
    for (_, r, c, h, w) in sample_tiles([((4096, 16384), None)], T, 16, seed=T):
        ref = oracle.ns_map(f64(X[r:r + h, c:c + w]), C32)
        got = f64(Y[r:r + h, c:c + w])
        assert rel(got, ref) <= TOL16
        assert svd_dev(got, ref) <= SVTOL


def sv_of(a):
    """Singular values of a wide fp64 matrix from the eigenvalues of a a^T."""
    ev = np.linalg.eigvalsh(a @ a.T)
    return np.sqrt(np.clip(ev, 0.0, None))[::-1]


def test_4096x16384_full_ns_against_oracle(hm):
    """Full NS of the whole 4096 x 16384 matrix (reductions 16384 deep) and of
    its transpose (the transpose trick), each against the fp64 oracle: relative
    Frobenius error <= 3e-2 and singular values within 0.05."""
    dev = torch.device("cuda", 0)
    X = inputs.gaussian_torch(4096, 16384, 3, dev)
    Xt = X.t().contiguous()
    Y, Yt = torch.empty_like(X), torch.empty_like(Xt)
    p = hm.params(0, QUINTIC, steps=5)
    hm.ns_full([X], [Y], p)
    hm.ns_full([Xt], [Yt], p)
    assert hm.device_status() == 0
    xin = f64(X)
    ref = oracle.ns_map(xin, C32)
    got, got_t = f64(Y), f64(Yt)
    del X, Xt, Y, Yt
    torch.cuda.empty_cache()
    assert rel(got, ref) <= TOL16
    assert rel(got_t.T, ref) <= TOL16
    sref = sv_of(ref)
    assert np.max(np.abs(sv_of(got) - sref)) <= SVTOL
    assert np.max(np.abs(sv_of(np.ascontiguousarray(got_t.T)) - sref)) <= SVTOL


def test_llama7b_update_out_T256_sampled_tiles(hm):
    """The 7B-shaped set at T = 256 (staged, chunks of at most 16 GB) on a
    2-layer slice, checking the update O itself against the oracle."""
    import bench
    dev = torch.device("cuda", 0)
    mats, W, M, G = bench.make_state(dev, seed_base=11, layers=2)
    splits = [s for _, s in mats]
    O = [torch.empty_like(x) for x in M]
    picks = sample_tiles(mats, 256, 24, seed=7)
    before = [(f64(M[i][r:r + h, c:c + w]), f64(G[i][r:r + h, c:c + w])) for (i, r, c, h, w) in picks]
    p = hm.params(256, QUINTIC, steps=5, chunk_bytes=16 << 30)
    hm.momentum_step(W, M, G, bench.MU, bench.LR, p, splits=splits, update_out=O)
    assert hm.device_status() == 0
    for (i, r, c, h, w), (m0, g0) in zip(picks, before):
        mp = oracle.momentum(m0, g0, bench.MU)
        assert np.all(np.abs(f64(M[i][r:r + h, c:c + w]) - mp) <= bf16_ulp(mp))
        ref = oracle.ns_map(mp, C32)
        got = f64(O[i][r:r + h, c:c + w])
        assert rel(got, ref) <= TOL16
        assert svd_dev(got, ref) <= SVTOL


def test_moe_experts_gram_and_standard_sampled(hm):
    """64 experts 1024 x 4096: Gram NS (fp16, restart at t = 3) and standard
    NS on all of them; two experts recomputed by the oracle."""
    dev = torch.device("cuda", 0)
    E = [inputs.low_rank_plus_noise_torch(1024, 4096, 1024, 0.001, 40 + i, dev, sigma="exp") for i in range(64)]
    Yg, Ys = [torch.empty_like(x) for x in E], [torch.empty_like(x) for x in E]
    hm.gram_ns(E, Yg, hm.params(0, QUINTIC, steps=5, compute=hm.FP16, restart=(3,)))
    hm.ns_full(E, Ys, hm.params(0, QUINTIC, steps=5))
    assert hm.device_status() == 0
    for k in (0, 37):
        ref = oracle.ns_map(f64(E[k]), C32)
        for Y in (Yg, Ys):
            got = f64(Y[k])
            assert rel(got, ref) <= TOL16
            assert svd_dev(got, ref) <= SVTOL


def test_gram_and_fp16_ns_2048x4096_against_oracle(hm):
    """One 2048 x 4096 matrix: Gram NS (fp16, restart at t = 3) and standard NS
    with fp16 operands.  At n >= 2048 the symmetric n x n products run on
    128 x 256 tiles, with Gram's fp32 terms kept on and below the diagonal,
    its Q in fp16, and fp16 NS's operand written by the second pass over the
    input; the 64-expert test (n = 1024) reaches none of that with 256-column
    tiles.  Both outputs are compared with the oracle's Gram NS, which equals
    its standard NS to ~1e-14 (pinned on the CPU)."""
    x = inputs.gaussian_torch(2048, 4096, 2048, "cuda")
    yg, ys = torch.empty_like(x), torch.empty_like(x)
    hm.gram_ns([x], [yg], hm.params(0, QUINTIC, steps=5, compute=hm.FP16, restart=(3,)))
    hm.ns_full([x], [ys], hm.params(0, QUINTIC, steps=5, compute=hm.FP16))
    assert hm.device_status() == 0
    ref = oracle.gram_ns(f64(x), C32, restart=(3,))
    for y in (yg, ys):
        got = f64(y)
        assert rel(got, ref) <= TOL16
        assert svd_dev(got, ref) <= SVTOL
