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


def test_device_timeout_is_reported_and_context_survives(hm):
    x = torch.from_numpy(inputs.gaussian((512, 512), seed=5)).to("cuda", torch.bfloat16)
    y = torch.empty_like(x)
    p = hm.params(128, inputs.QUINTIC, steps=5)
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
    ref = oracle.ns_tiled(x.double().cpu().numpy(), 128, [inputs.QUINTIC] * 5)
    assert per_tile_errors(y.double().cpu().numpy(), ref, 128).max() <= 3e-2
