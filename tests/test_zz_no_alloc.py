"""GPU test of himuon_ns_static, the entry point that allocates nothing.

Callers that cannot allocate device memory (a memory pool that owns all of
HBM, a runtime that forbids cudaMalloc/cudaFree inside training steps) use
himuon_ns_static, whose scratch is a fixed 32 MiB device array inside the
library.  This file checks, through the C ABI, that two calls in a row give
the same results as the workspace-taking entry points on the same inputs,
within the tensor-core path's per-tile tolerance (3e-2 relative Frobenius
error; the arithmetic is the same, so the results in fact agree far closer),
that the array's leftover contents from one call do not leak into the next
(the second call has zero-padded ragged tiles), and that a call too large
for the array is refused before anything is enqueued.

It runs last (file name) so that a failing first-failure run has already run
every other test, and passes both alone and after the other tests.
"""
import numpy as np
import pytest

from tests.parity_util import per_tile_errors
from tiled_newton_schulz_b200 import inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 3e-2


@pytest.fixture(scope="module")
def hm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_newton_schulz_b200 import himuon
    himuon.load()
    return himuon


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda", torch.bfloat16)


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def test_static_scratch_matches_workspace_path_twice(hm):
    # call 1: full-matrix NS of two matrices (one needs zero padding)
    xs = [bf16(inputs.gaussian((384, 640), seed=41)), bf16(inputs.gaussian((300, 500), seed=42))]
    p_full = hm.params(0, inputs.QUINTIC, steps=5, compute=hm.BF16)
    ref = [torch.empty_like(x) for x in xs]
    hm.ns_full(xs, ref, p_full)
    got = [torch.full_like(x, float("nan")) for x in xs]
    assert hm.ns_static(xs, got, p_full) == 0
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        a, b = f64(g), f64(r)
        assert np.all(np.isfinite(a))
        assert per_tile_errors(a, b, 0).max() <= TOL
    # call 2: tiled NS with T = 256 on a ragged matrix (padded edge tiles)
    y = bf16(inputs.gaussian((600, 520), seed=43))
    p256 = hm.params(256, inputs.QUINTIC, steps=5, compute=hm.BF16)
    ref2 = torch.empty_like(y)
    hm.ns_tiled([y], [ref2], p256)
    got2 = torch.full_like(y, float("nan"))
    assert hm.ns_static([y], [got2], p256) == 0
    torch.cuda.synchronize()
    a, b = f64(got2), f64(ref2)
    assert np.all(np.isfinite(a))
    assert per_tile_errors(a, b, 256).max() <= TOL
    assert hm.device_status() == 0


def test_static_scratch_fp32_matches_workspace_path(hm):
    """An fp32 call (CUDA-core path, its own workspace layout): 256 x 512 at
    T = 256 and full NS, against the workspace entry points within the fp32
    path's tolerance (1e-4 per-tile relative Frobenius error)."""
    x = torch.from_numpy(inputs.gaussian((256, 512), seed=44)).to("cuda", torch.float32)
    for T in (256, 0):
        p = hm.params(T, inputs.QUINTIC, steps=5, compute=hm.FP32)
        ref = torch.empty_like(x)
        (hm.ns_tiled if T > 0 else hm.ns_full)([x], [ref], p)
        got = torch.full_like(x, float("nan"))
        assert hm.ns_static([x], [got], p) == 0
        torch.cuda.synchronize()
        a, b = got.double().cpu().numpy(), ref.double().cpu().numpy()
        assert np.all(np.isfinite(a))
        assert per_tile_errors(a, b, T).max() <= 1e-4
    assert hm.device_status() == 0


def test_static_scratch_refuses_oversized_calls(hm):
    x = torch.zeros(4096, 4096, device="cuda", dtype=torch.bfloat16)
    out = torch.zeros_like(x)
    before = hm.launch_count()
    rc = hm.ns_static([x], [out], hm.params(0, inputs.QUINTIC, steps=5))
    assert rc == hm.ERR_TOO_LARGE
    assert "scratch" in hm.status_string(rc)
    assert hm.launch_count() == before
