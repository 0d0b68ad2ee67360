"""Failure detection without a GPU fault (needs a B200).

Every wait inside the kernels is bounded in time (two seconds).  A wait that
runs out records HIMUON_ERR_TIMEOUT in the device status word, the CTA stops
its work after waiting (bounded) for its own copies and MMAs in flight, frees
its tensor memory and returns; the host reads the status with
himuon_get_device_status().  HIMUON_TEST_STALL=1 makes one tile group wait on
a barrier that nothing arrives on, so the timeout path runs for real; the
context must stay usable and the next call must be correct.
"""
import os

import numpy as np
import pytest

import oracle
from tests.parity_util import per_tile_errors
from tiled_newton_schulz_b200 import inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_newton_schulz_b200 import himuon
    himuon.load()
    return himuon


@pytest.mark.parametrize("T", [128, 256])
def test_device_timeout_is_reported_and_context_survives(hm, T):
    """T = 128 runs the one-CTA kernel, T = 256 the CTA-pair kernel."""
    x = torch.from_numpy(inputs.gaussian((512, 512), seed=5)).to("cuda", torch.bfloat16)
    y = torch.empty_like(x)
    p = hm.params(T, inputs.QUINTIC, steps=5)
    assert hm.device_status() == 0
    os.environ["HIMUON_TEST_STALL"] = "1"
    try:
        hm.ns_tiled([x], [y], p)
        status = hm.device_status()
    finally:
        del os.environ["HIMUON_TEST_STALL"]
    assert status == -6, hm.status_string(status)          # HIMUON_ERR_TIMEOUT
    assert hm.device_status() == 0                           # reading clears it
    # the context is still usable and the next call is right
    hm.ns_tiled([x], [y], p)
    assert hm.device_status() == 0
    ref = oracle.ns_tiled(x.double().cpu().numpy(), T, [inputs.QUINTIC] * 5)
    assert per_tile_errors(y.double().cpu().numpy(), ref, T).max() <= 3e-2


def test_undersized_or_misaligned_workspace_is_refused_before_any_launch(hm):
    """A staged call (T = 512) with too small or badly aligned scratch returns
    HIMUON_ERR_WORKSPACE / HIMUON_ERR_ALIGNMENT before enqueuing a kernel; so
    does a call with per-matrix tile sizes whose second group lacks scratch,
    although its first group (on chip) needs none."""
    import ctypes
    x = torch.from_numpy(inputs.gaussian((512, 512), seed=6)).to("cuda", torch.bfloat16)
    y = torch.empty_like(x)
    p = hm.params(512, inputs.QUINTIC, steps=5)
    need = hm.workspace_size([x], p, hm.OP_NS_TILED)
    assert need > 4096
    n0 = hm.launch_count()
    with pytest.raises(hm.HimuonError) as e:
        hm.ns_tiled([x], [y], p, workspace=torch.empty(1024, dtype=torch.uint8, device="cuda"))
    assert e.value.code == -3                                # HIMUON_ERR_WORKSPACE
    big = torch.empty(need + 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(hm.HimuonError) as e:
        hm.ns_tiled([x], [y], p, workspace=big[16:])         # 16 bytes past a 256-byte boundary
    assert e.value.code == -4                                # HIMUON_ERR_ALIGNMENT
    lib = hm.load()
    assert lib.himuon_ns_tiled(hm._mats([x]), hm._mats([y]), 1, None, ctypes.byref(p), None, 0, None) == -3
    x2, y2 = x.clone(), torch.empty_like(x)
    pt = hm.params(128, inputs.QUINTIC, steps=5, tiles=[128, 512])
    with pytest.raises(hm.HimuonError) as e:
        hm.ns_tiled([x2, x], [y2, y], pt, workspace=torch.empty(1024, dtype=torch.uint8, device="cuda"))
    assert e.value.code == -3
    assert hm.launch_count() == n0                           # nothing was enqueued
    assert hm.device_status() == 0
    hm.ns_tiled([x], [y], p, workspace=big[:need])           # the right size and alignment run
    assert hm.device_status() == 0 and hm.launch_count() > n0
    ref = oracle.ns_tiled(x.double().cpu().numpy(), 512, [inputs.QUINTIC] * 5)
    assert per_tile_errors(y.double().cpu().numpy(), ref, 512).max() <= 3e-2
