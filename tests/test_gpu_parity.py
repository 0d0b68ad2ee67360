"""GPU parity of the CUDA path against the fp64 oracle (needs a B200).

Every case draws seeded inputs, rounds them to the storage dtype, feeds the
identical values to the library (through the C ABI) and to the oracle, and
compares element by element.

Tolerances (stated for the two arithmetic paths):
* fp32 CUDA-core path: per-tile relative Frobenius error <= 1e-4.
* bf16/fp16 tensor-core path: per-tile relative Frobenius error <= 3e-2, and
  sorted singular values of every checked tile within 0.05 of the oracle's,
  for every tile size and shape, ragged edges included.  (A bf16 call rounds
  the operands of tiles with a short side of at most 64 to fp16 on chip and
  runs such tiles in fp32 when staged: with bf16 operands their singular
  values move by up to ~0.1 in a CPU emulation of the kernel's arithmetic.)
* the stored momentum M' = mu M + G: within one bf16 ulp of the fp64 value.
* tile placement: bit-exact (integer-coded tiles).
"""
import numpy as np
import pytest

import oracle
from tests.parity_util import bf16_ulp, max_sv_diff, per_tile_errors, tiles, to_np
from tiled_newton_schulz_b200 import inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

QUINTIC = inputs.QUINTIC
C32 = [tuple(float(np.float32(v)) for v in QUINTIC)] * 5   # the fp32 values the library receives
TOL16, TOL32, SVTOL = 3e-2, 1e-4, 0.05


@pytest.fixture(scope="module")
def hm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_newton_schulz_b200 import himuon
    himuon.load()
    return himuon


def dev(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dtype)


def check16(Y, Yref, T, sv_sample=64):
    """Per-tile relative Frobenius error <= 3e-2 and singular values within
    0.05 on (a sample of) the tiles, for either 16-bit operand type."""
    err = per_tile_errors(Y, Yref, T)
    assert np.all(err <= TOL16), f"max per-tile rel err {err.max():.4g}"
    sv = max_sv_diff(Y, Yref, T, sample=sv_sample)
    assert sv <= SVTOL, f"max singular-value deviation {sv:.4g}"
    return err.max()


def run_ns(hm, X, T, compute, dtype, full=False):
    x = dev(X, dtype)
    y = torch.empty_like(x)
    p = hm.params(T, QUINTIC, steps=5, compute=compute)
    (hm.ns_full if full else hm.ns_tiled)([x], [y], p)
    assert hm.device_status() == 0
    return to_np(x), to_np(y)


@pytest.mark.parametrize("compute", ["bf16", "fp16"])
@pytest.mark.parametrize("H,W", [(256, 384), (300, 500), (128, 128), (100, 70), (1, 300)])
def test_resident_tiled_ns(hm, H, W, compute):
    X = inputs.gaussian((H, W), seed=H + W)
    code = hm.BF16 if compute == "bf16" else hm.FP16
    xin, y = run_ns(hm, X, 128, code, torch.bfloat16)
    check16(y, oracle.ns_tiled(xin, 128, C32), 128)


# Step lists for the on-chip kernel's scaled operand: the pages' quintic step,
# the textbook cubic Newton-Schulz step (c = 0: the operand is not rescaled and
# S is zero) and an odd quintic with b = 0 (MMA2 overwrites instead of
# accumulating); mixing them makes the operand scale change between steps.
QUINTIC_T = tuple(QUINTIC)
CUBIC = (1.5, -0.5, 0.0)
NO_B = (1.5, 0.0, -0.5)
# Sixteen steps (the maximum) end in cubic steps, which contract towards the
# polar factor: sixteen quintic steps do not contract, and their bf16 operand
# roundings add up past the 3e-2 budget (an emulation of exactly the kernel's
# rounding points gives 5.2% bf16 / 3.1% fp16 per tile for them, 2.3% / 0.5%
# for this list; the GPU matched the emulation).  This list also multiplies a
# singular value near zero by about 4e4 (3.4445^5 x 1.5^11), so the noise
# floor of a low-rank-plus-noise tile ends in the steep middle of the map,
# where an 8-bit operand rounding moves it by ~0.25 (bf16; fp16 keeps it
# within 0.05; tests/test_rounding_budget.py): its cases run fp16 operands.
STEP_LISTS = {
    "K1": [QUINTIC_T],
    "K16": [QUINTIC_T] * 5 + [CUBIC] * 11,
    "mixed": [QUINTIC_T, CUBIC, NO_B, (2.0, -1.5, 0.5), QUINTIC_T, CUBIC],
}


@pytest.mark.parametrize("compute", ["bf16", "fp16"])
@pytest.mark.parametrize("T", [128, 64])
@pytest.mark.parametrize("steps", sorted(STEP_LISTS))
def test_resident_step_lists(hm, steps, T, compute):
    """One step, the maximum of sixteen, and a list whose coefficients change
    from step to step (including c = 0 and b = 0), on the on-chip kernel."""
    X = inputs.low_rank_plus_noise(256, 384, inputs.sigma_inverse(32), 0.01, seed=T + len(steps))
    co = STEP_LISTS[steps]
    x = dev(X, torch.bfloat16)
    y = torch.empty_like(x)
    code = hm.BF16 if (compute == "bf16" and steps != "K16") else hm.FP16
    hm.ns_tiled([x], [y], hm.params(T, co, compute=code))
    assert hm.device_status() == 0
    c32 = [tuple(float(np.float32(v)) for v in tri) for tri in co]
    check16(to_np(y), oracle.ns_tiled(to_np(x), T, c32), T)


@pytest.mark.parametrize("steps", ["mixed", "K1"])
def test_momentum_step_step_lists(hm, steps):
    """The fused step (momentum prologue, W update and O out) with a step list
    whose last step sets the output scale differently from the first."""
    co = STEP_LISTS[steps]
    H, W = 256, 384
    w = dev(0.02 * inputs.gaussian((H, W), seed=3), torch.bfloat16)
    m = dev(inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=4), torch.bfloat16)
    g = dev(inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=5), torch.bfloat16)
    o = torch.empty_like(m)
    w0, m0, g0 = to_np(w), to_np(m), to_np(g)
    hm.momentum_step([w], [m], [g], 0.95, 0.02, hm.params(128, co), update_out=[o])
    assert hm.device_status() == 0
    c32 = [tuple(float(np.float32(v)) for v in tri) for tri in co]
    W2, M2, O = oracle.momentum_step(w0, m0, g0, 0.95, 0.02, 128, c32)
    assert np.all(np.abs(to_np(m) - M2) <= bf16_ulp(M2))
    check16(to_np(o), O, 128)
    bound = np.linalg.norm(0.5 * bf16_ulp(W2)) + float(np.float32(0.02)) * TOL16 * np.linalg.norm(O)
    assert np.linalg.norm(to_np(w) - W2) <= bound


@pytest.mark.parametrize("compute", ["bf16", "fp16"])
@pytest.mark.parametrize("T", [32, 64])
@pytest.mark.parametrize("H,W", [(256, 384), (300, 500), (100, 70), (33, 65), (128, 4096)])
def test_resident_packed_small_tiles(hm, H, W, T, compute):
    """T = 64 / 32: two / four tiles share one 128 x 128 super-tile as diagonal blocks."""
    X = inputs.gaussian((H, W), seed=7 * H + W + T)
    code = hm.BF16 if compute == "bf16" else hm.FP16
    xin, y = run_ns(hm, X, T, code, torch.bfloat16)
    check16(y, oracle.ns_tiled(xin, T, C32), T)


@pytest.mark.parametrize("T", [32, 64])
def test_momentum_step_packed_small_tiles(hm, T):
    rng = np.random.default_rng(T)
    shapes = [(192, 320), (96, 128), (64, 33)]
    w = [dev(0.02 * rng.standard_normal(sh), torch.bfloat16) for sh in shapes]
    m = [dev(inputs.low_rank_plus_noise(*sh, inputs.sigma_inverse(8), 0.01, seed=300 + i), torch.bfloat16)
         for i, sh in enumerate(shapes)]
    g = [dev(inputs.low_rank_plus_noise(*sh, inputs.sigma_inverse(8), 0.01, seed=400 + i), torch.bfloat16)
         for i, sh in enumerate(shapes)]
    o = [torch.empty_like(x) for x in m]
    w0, m0, g0 = [to_np(x) for x in w], [to_np(x) for x in m], [to_np(x) for x in g]
    hm.momentum_step(w, m, g, 0.95, 0.02, hm.params(T, QUINTIC, steps=5, compute=hm.FP16), update_out=o)
    assert hm.device_status() == 0
    for i in range(len(shapes)):
        W2, M2, O = oracle.momentum_step(w0[i], m0[i], g0[i], 0.95, 0.02, T, C32)
        assert np.all(np.abs(to_np(m[i]) - M2) <= bf16_ulp(M2))
        check16(to_np(o[i]), O, T)
        wg = to_np(w[i])
        bound = np.linalg.norm(0.5 * bf16_ulp(W2)) + float(np.float32(0.02)) * TOL16 * np.linalg.norm(O)
        assert np.linalg.norm(wg - W2) <= bound


def test_resident_zero_tile_and_scale(hm):
    X = inputs.gaussian((256, 256), seed=7)
    X[:128, 128:] = 0.0                         # one all-zero tile
    X[128:, :128] *= 1e-6                        # one tiny tile
    X[128:, 128:] *= 1e3                         # one large tile
    xin, y = run_ns(hm, X, 128, hm.BF16, torch.bfloat16)
    assert np.all(y[:128, 128:] == 0.0)
    check16(y, oracle.ns_tiled(xin, 128, C32), 128)


@pytest.mark.parametrize("T", [64, 128, 256, 512])
def test_fp32_path_small_matrix(hm, T):
    """256 x 512 fp32, i.i.d. N(0,1) from seed 0, fp32 arithmetic."""
    X = inputs.gaussian((256, 512), seed=0)
    xin, y = run_ns(hm, X, T, hm.FP32, torch.float32)
    err = per_tile_errors(y, oracle.ns_tiled(xin, T, C32), T)
    assert err.max() <= TOL32, err.max()


def test_fp32_path_large_T_is_full_ns(hm):
    X = inputs.gaussian((256, 512), seed=0)
    xin, y = run_ns(hm, X, 512, hm.FP32, torch.float32)
    _, yf = run_ns(hm, X, 0, hm.FP32, torch.float32, full=True)
    ref = oracle.ns_map(xin, C32)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) <= TOL32
    assert np.linalg.norm(yf - ref) / np.linalg.norm(ref) <= TOL32


@pytest.mark.parametrize("compute", ["bf16", "fp16"])
@pytest.mark.parametrize("H,W,T", [(512, 768, 256), (600, 520, 256), (512, 1024, 512)])
def test_staged_tiled_ns(hm, H, W, T, compute):
    X = inputs.gaussian((H, W), seed=H * 3 + W + T)
    code = hm.BF16 if compute == "bf16" else hm.FP16
    xin, y = run_ns(hm, X, T, code, torch.bfloat16)
    check16(y, oracle.ns_tiled(xin, T, C32), T)


@pytest.mark.parametrize("H,W", [(256, 1024), (1024, 256), (300, 700)])
def test_full_ns_bf16_with_transpose(hm, H, W):
    X = inputs.gaussian((H, W), seed=H + 2 * W)
    xin, y = run_ns(hm, X, 0, hm.BF16, torch.bfloat16, full=True)
    check16(y, oracle.ns_map(xin, C32), 0)


@pytest.mark.parametrize("dtype", ["float32", "float16"])
@pytest.mark.parametrize("H,W,T", [(300, 700, 0), (700, 300, 0), (600, 520, 512), (520, 600, 512)])
def test_staged_16bit_compute_io_dtypes(hm, H, W, T, dtype):
    """16-bit operands with fp32 or fp16 inputs and outputs on the staged path,
    whose last product writes the caller's buffer from its epilogue: straight
    and transposed tiles, ragged edges (600 x 520 at T = 512 has 88-wide and
    88-high tiles)."""
    X = inputs.gaussian((H, W), seed=H + 5 * W + T)
    xin, y = run_ns(hm, X, T, hm.BF16, getattr(torch, dtype), full=T == 0)
    ref = oracle.ns_map(xin, C32) if T == 0 else oracle.ns_tiled(xin, T, C32)
    check16(y, ref, T)


def test_staged_momentum_step_fp32_w_and_update_out(hm):
    """The staged momentum step (T = 512, ragged and transposed tiles) with an
    fp32 W and a bf16 update output: O matches the oracle per tile and
    W' = W - lr O within lr times O's tolerance (fp32 W adds no rounding of
    note)."""
    H, W, T, lr = 700, 600, 512, 0.02
    w0 = 0.02 * inputs.gaussian((H, W), seed=11)
    m0 = inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=12)
    g0 = inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=13)
    w, m, g = dev(w0, torch.float32), dev(m0, torch.bfloat16), dev(g0, torch.bfloat16)
    o = torch.empty_like(m)
    mi, gi, wi = to_np(m), to_np(g), to_np(w)
    hm.momentum_step([w], [m], [g], 0.95, lr, hm.params(T, QUINTIC, steps=5), update_out=[o])
    assert hm.device_status() == 0
    W2, _, O = oracle.momentum_step(wi, mi, gi, 0.95, lr, T, C32)
    check16(to_np(o), O, T)
    assert np.linalg.norm(to_np(w) - W2) <= float(np.float32(lr)) * TOL16 * np.linalg.norm(O)


def test_momentum_step_resident(hm):
    shapes = [(256, 256), (256, 512), (384, 128)]
    rng = np.random.default_rng(12)
    Ws, Ms, Gs = [], [], []
    for i, (H, W) in enumerate(shapes):
        Ws.append(0.02 * rng.standard_normal((H, W)))
        Ms.append(inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=100 + i))
        Gs.append(inputs.low_rank_plus_noise(H, W, inputs.sigma_inverse(16), 0.01, seed=200 + i))
    w = [dev(x, torch.bfloat16) for x in Ws]
    m = [dev(x, torch.bfloat16) for x in Ms]
    g = [dev(x, torch.bfloat16) for x in Gs]
    o = [torch.empty_like(x) for x in m]
    w0, m0, g0 = [to_np(x) for x in w], [to_np(x) for x in m], [to_np(x) for x in g]
    mu, lr = 0.95, 0.02
    hm.momentum_step(w, m, g, mu, lr, hm.params(128, QUINTIC, steps=5), update_out=o)
    assert hm.device_status() == 0
    for i in range(len(shapes)):
        W2, M2, O = oracle.momentum_step(w0[i], m0[i], g0[i], mu, lr, 128, C32)
        mg = to_np(m[i])
        assert np.all(np.abs(mg - M2) <= bf16_ulp(M2)), "M' beyond one bf16 ulp"
        check16(to_np(o[i]), O, 128)
        # W' = W - lr O: bf16 rounding of W' plus lr times the NS error
        wg = to_np(w[i])
        for r0 in range(0, M2.shape[0], 128):
            for c0 in range(0, M2.shape[1], 128):
                sl = np.s_[r0:r0 + 128, c0:c0 + 128]
                bound = np.linalg.norm(0.5 * bf16_ulp(W2[sl])) + float(np.float32(lr)) * TOL16 * np.linalg.norm(O[sl])
                assert np.linalg.norm(wg[sl] - W2[sl]) <= bound


@pytest.mark.parametrize("T", [32, 64, 128, 256])
def test_integer_coded_reassembly_bitexact(hm, T):
    """Tile t holds c_t P_t (signed permutation with its own shift and signs);
    the output keeps support and signs exactly, so any misplaced, swapped or
    transposed tile fails."""
    H, W = (512, 384) if T < 256 else (768, 640)
    X = np.zeros((H, W))
    for t, (r0, c0, h, w) in enumerate(oracle.tile_grid(H, W, T)):
        P = inputs.signed_permutation(T, shift=(7 * t) % T, sign_bits=(t * 2654435761) & 0x7FFFFFFF)
        X[r0:r0 + h, c0:c0 + w] = (0.5 + 0.25 * t) * P[:h, :w]
    xin, y = run_ns(hm, X, T, hm.BF16, torch.bfloat16)
    assert np.array_equal(np.sign(y), np.sign(xin))


@pytest.mark.parametrize("restart", [(3,), (), (2, 4), (2, 3), (1,)])
def test_gram_ns_fp16(hm, restart):
    n, m = 256, 1024
    X = inputs.low_rank_plus_noise(n, m, inputs.sigma_exp(n, 32.0), 1e-3, seed=4)
    x = dev(X, torch.bfloat16)
    y = torch.empty_like(x)
    hm.gram_ns([x], [y], hm.params(0, QUINTIC, steps=5, compute=hm.FP16, restart=restart))
    assert hm.device_status() == 0
    xin = to_np(x)
    ref = oracle.gram_ns(xin, C32, restart=restart)
    yy = to_np(y)
    assert np.linalg.norm(yy - ref) / np.linalg.norm(ref) <= TOL16
    assert max_sv_diff(yy, ref, 0) <= SVTOL


@pytest.mark.parametrize("restart", [(3,), (2, 4)])
def test_gram_ns_fp32(hm, restart):
    """Gram NS with fp32 storage and arithmetic (CUDA-core products) against
    the oracle within the fp32 tolerance; restarts before steps 3, or 2 and 4."""
    X = inputs.gaussian((256, 1024), seed=41)
    x = dev(X, torch.float32)
    y = torch.empty_like(x)
    hm.gram_ns([x], [y], hm.params(0, QUINTIC, steps=5, compute=hm.FP32, restart=restart))
    assert hm.device_status() == 0
    ref = oracle.gram_ns(to_np(x), C32, restart=restart)
    assert np.linalg.norm(to_np(y) - ref) / np.linalg.norm(ref) <= TOL32


@pytest.mark.parametrize("T", [128, 256])
def test_gram_ns_tiled_fp16(hm, T):
    """Gram NS applied per tile (ragged edge rows and columns), fp16 operands,
    restart at t = 3, against the oracle's tile-by-tile Gram NS."""
    H, W = 640, 832
    X = inputs.low_rank_plus_noise(H, W, inputs.sigma_exp(H, 32.0), 1e-3, seed=12)
    x = dev(X, torch.bfloat16)
    y = torch.empty_like(x)
    hm.gram_ns([x], [y], hm.params(T, QUINTIC, steps=5, compute=hm.FP16, restart=(3,)))
    assert hm.device_status() == 0
    xin = to_np(x)
    ref = oracle.gram_ns_tiled(xin, T, C32, restart=(3,))
    yy = to_np(y)
    for r0, c0, h, w in oracle.tile_grid(H, W, T):
        sl = np.s_[r0:r0 + h, c0:c0 + w]
        assert np.linalg.norm(yy[sl] - ref[sl]) / np.linalg.norm(ref[sl]) <= TOL16
        assert max_sv_diff(yy[sl], ref[sl], 0) <= SVTOL


def test_split_qkv_blocks(hm):
    """A fused 256 x 768 tensor split into three 256 x 256 blocks before full NS."""
    X = inputs.gaussian((256, 768), seed=31)
    x = dev(X, torch.bfloat16)
    y = torch.empty_like(x)
    split = [(1, (256, 256, 256))]
    hm.ns_full([x], [y], hm.params(0, QUINTIC, steps=5), splits=split)
    xin = to_np(x)
    ref = oracle.ns_tiled_split(xin, 0 or 10 ** 9, C32, split=split[0])
    yy = to_np(y)
    for j in range(3):
        sl = np.s_[:, 256 * j:256 * (j + 1)]
        assert np.linalg.norm(yy[sl] - ref[sl]) / np.linalg.norm(ref[sl]) <= TOL16


# Safety factor ("Gram Newton-Schulz" page, sec. 6 implementation notes: the
# normalised input divided by 1.05), on chip, staged, full NS and Gram NS.
@pytest.mark.parametrize("T,H,W", [(128, 256, 384), (64, 256, 384), (256, 512, 768), (0, 256, 1024)])
def test_safety_factor(hm, T, H, W):
    X = inputs.gaussian((H, W), seed=H + W + T + 1)
    x = dev(X, torch.bfloat16)
    y = torch.empty_like(x)
    co = [QUINTIC_T, (2.9, -3.1, 1.1)]          # two steps keep the factor visible
    p = hm.params(T, co, compute=hm.FP16, safety=1.05)
    (hm.ns_tiled if T > 0 else hm.ns_full)([x], [y], p)
    assert hm.device_status() == 0
    xin = to_np(x)
    c32 = [tuple(float(np.float32(v)) for v in tri) for tri in co]
    s32 = float(np.float32(1.05))
    ref = oracle.ns_tiled(xin, T if T > 0 else 10 ** 9, c32, safety=s32)
    check16(to_np(y), ref, T)
    off = oracle.ns_tiled(xin, T if T > 0 else 10 ** 9, c32)
    assert np.linalg.norm(to_np(y) - off) > 3 * np.linalg.norm(to_np(y) - ref)


def test_gram_ns_safety_factor(hm):
    X = inputs.low_rank_plus_noise(256, 1024, inputs.sigma_exp(256, 32.0), 1e-3, seed=8)
    x = dev(X, torch.bfloat16)
    y = torch.empty_like(x)
    co = [QUINTIC_T, (2.9, -3.1, 1.1)]
    hm.gram_ns([x], [y], hm.params(0, co, compute=hm.FP16, safety=1.05, restart=(2,)))
    assert hm.device_status() == 0
    c32 = [tuple(float(np.float32(v)) for v in tri) for tri in co]
    ref = oracle.gram_ns(to_np(x), c32, restart=(2,), safety=float(np.float32(1.05)))
    yy = to_np(y)
    assert np.linalg.norm(yy - ref) / np.linalg.norm(ref) <= TOL16
    assert max_sv_diff(yy, ref, 0) <= SVTOL


# Gram NS with a coefficient triple per step (the page's Algorithm 3 indexes
# a_t, b_t, c_t by the step), restarts included.
GRAM_STEPS = [QUINTIC_T, (2.9, -3.1, 1.1), (2.2, -1.6, 0.45), (1.9, -1.3, 0.4), (1.6, -0.8, 0.2)]


@pytest.mark.parametrize("restart", [(3,), (), (2, 4)])
@pytest.mark.parametrize("T", [0, 128])
def test_gram_ns_per_step_coefficients(hm, restart, T):
    H, W = (256, 1024) if T == 0 else (384, 640)
    X = inputs.low_rank_plus_noise(H, W, inputs.sigma_exp(min(H, W), 32.0), 1e-3, seed=9 + T)
    x = dev(X, torch.bfloat16)
    y = torch.empty_like(x)
    hm.gram_ns([x], [y], hm.params(T, GRAM_STEPS, compute=hm.FP16, restart=restart))
    assert hm.device_status() == 0
    c32 = [tuple(float(np.float32(v)) for v in tri) for tri in GRAM_STEPS]
    ref = oracle.gram_ns_tiled(to_np(x), T, c32, restart=restart)
    check16(to_np(y), ref, T)


# T = 256 on a CTA pair: every 256 x 256 tile is split by rows over two CTAs.
@pytest.mark.parametrize("compute", ["bf16", "fp16"])
@pytest.mark.parametrize("H,W", [(512, 768), (600, 520), (256, 256), (100, 70), (700, 300), (1, 300), (130, 1000)])
def test_pair_tiled_ns(hm, H, W, compute):
    """Ragged edges in both directions, a tile whose second CTA holds only
    padding (100 x 70, 130 rows), tall tiles, and thin tiles that take fp16
    operands in a bf16 call (1 x 300)."""
    X = inputs.gaussian((H, W), seed=11 * H + W)
    code = hm.BF16 if compute == "bf16" else hm.FP16
    xin, y = run_ns(hm, X, 256, code, torch.bfloat16)
    check16(y, oracle.ns_tiled(xin, 256, C32), 256)


@pytest.mark.parametrize("steps", sorted(STEP_LISTS))
def test_pair_step_lists(hm, steps):
    X = inputs.low_rank_plus_noise(512, 768, inputs.sigma_inverse(32), 0.01, seed=3 + len(steps))
    co = STEP_LISTS[steps]
    x = dev(X, torch.bfloat16)
    y = torch.empty_like(x)
    hm.ns_tiled([x], [y], hm.params(256, co, compute=hm.FP16 if steps == "K16" else hm.BF16))
    assert hm.device_status() == 0
    c32 = [tuple(float(np.float32(v)) for v in tri) for tri in co]
    check16(to_np(y), oracle.ns_tiled(to_np(x), 256, c32), 256)


def test_pair_momentum_step(hm):
    """The fused step on the pair kernel: M' within one bf16 ulp, O against
    the oracle, W' = W - lr O."""
    shapes = [(512, 512), (300, 700), (768, 256)]
    rng = np.random.default_rng(21)
    w = [dev(0.02 * rng.standard_normal(sh), torch.bfloat16) for sh in shapes]
    m = [dev(inputs.low_rank_plus_noise(*sh, inputs.sigma_inverse(16), 0.01, seed=500 + i), torch.bfloat16)
         for i, sh in enumerate(shapes)]
    g = [dev(inputs.low_rank_plus_noise(*sh, inputs.sigma_inverse(16), 0.01, seed=600 + i), torch.bfloat16)
         for i, sh in enumerate(shapes)]
    o = [torch.empty_like(x) for x in m]
    w0, m0, g0 = [to_np(x) for x in w], [to_np(x) for x in m], [to_np(x) for x in g]
    hm.momentum_step(w, m, g, 0.95, 0.02, hm.params(256, QUINTIC, steps=5), update_out=o)
    assert hm.device_status() == 0
    lr32 = float(np.float32(0.02))
    for i in range(len(shapes)):
        W2, M2, O = oracle.momentum_step(w0[i], m0[i], g0[i], 0.95, 0.02, 256, C32)
        assert np.all(np.abs(to_np(m[i]) - M2) <= bf16_ulp(M2))
        check16(to_np(o[i]), O, 256)
        got = to_np(o[i])
        wexp = w0[i] - lr32 * got
        assert np.all(np.abs(to_np(w[i]) - wexp) <= bf16_ulp(wexp) + lr32 * bf16_ulp(got) + 1e-12)


# ---- many tiles per CTA (pair): the loop over tiles, with the next tile's
# loads in flight during the current tile's last step
LOOP_SHAPES = [(520, 600), (40, 700), (300, 130)]   # ragged, thin (fp16 operands in bf16 calls), tall
_LOOP_REF = {}


def _loop_inputs():
    rng = np.random.default_rng(31)
    w = [0.02 * rng.standard_normal(sh) for sh in LOOP_SHAPES]
    m = [inputs.low_rank_plus_noise(*sh, inputs.sigma_inverse(16), 0.01, seed=700 + i) for i, sh in enumerate(LOOP_SHAPES)]
    g = [inputs.low_rank_plus_noise(*sh, inputs.sigma_inverse(16), 0.01, seed=800 + i) for i, sh in enumerate(LOOP_SHAPES)]
    bf = lambda a: to_np(torch.from_numpy(a).to(torch.bfloat16))
    return [bf(x) for x in w], [bf(x) for x in m], [bf(x) for x in g]


def _loop_reference(T, mode):
    key = (T, mode)
    if key not in _LOOP_REF:
        w0, m0, g0 = _loop_inputs()
        if mode == "ns":
            _LOOP_REF[key] = [oracle.ns_tiled(x, T, C32) for x in m0]
        else:
            _LOOP_REF[key] = [oracle.momentum_step(w0[i], m0[i], g0[i], 0.95, 0.02, T, C32)
                              for i in range(len(LOOP_SHAPES))]
    return _LOOP_REF[key]


@pytest.mark.parametrize("mode", ["ns", "step", "step_out"])
@pytest.mark.parametrize("T,ctas", [(256, 2), (256, 6), (128, 1), (128, 3), (64, 1), (64, 3), (32, 2)])
def test_onchip_tile_loop(hm, monkeypatch, T, ctas, mode):
    """HIMUON_MAX_CTAS caps the launch so that every CTA (pair) runs many
    tiles of three matrices in its loop: tile coordinates, loads issued
    during the previous tile's last step, per-tile operand type (the thin
    matrix's tiles take fp16 operands), ragged edges and the fused step's
    three outputs must all follow the tile being processed."""
    monkeypatch.setenv("HIMUON_MAX_CTAS", str(ctas))
    w0, m0, g0 = _loop_inputs()
    ref = _loop_reference(T, "ns" if mode == "ns" else "step")
    p = hm.params(T, QUINTIC, steps=5)
    if mode == "ns":
        x = [dev(a, torch.bfloat16) for a in m0]
        y = [torch.empty_like(a) for a in x]
        hm.ns_tiled(x, y, p)
        assert hm.device_status() == 0
        for i in range(len(LOOP_SHAPES)):
            check16(to_np(y[i]), ref[i], T)
        return
    w = [dev(a, torch.bfloat16) for a in w0]
    m = [dev(a, torch.bfloat16) for a in m0]
    g = [dev(a, torch.bfloat16) for a in g0]
    o = [torch.empty_like(a) for a in m] if mode == "step_out" else None
    hm.momentum_step(w, m, g, 0.95, 0.02, p, update_out=o)
    assert hm.device_status() == 0
    lr32 = float(np.float32(0.02))
    for i in range(len(LOOP_SHAPES)):
        W2, M2, O = ref[i]
        assert np.all(np.abs(to_np(m[i]) - M2) <= bf16_ulp(M2)), i
        wg = to_np(w[i])
        if o is not None:
            got = to_np(o[i])
            check16(got, O, T)
            wexp = w0[i] - lr32 * got
            assert np.all(np.abs(wg - wexp) <= bf16_ulp(wexp) + lr32 * bf16_ulp(got) + 1e-12)
        else:
            for (r, c, h, ww) in tiles(*LOOP_SHAPES[i], T):
                sl = np.s_[r:r + h, c:c + ww]
                bound = np.linalg.norm(0.5 * bf16_ulp(W2[sl])) + lr32 * TOL16 * np.linalg.norm(O[sl])
                assert np.linalg.norm(wg[sl] - W2[sl]) <= bound, (i, r, c)
