"""The flat sharded Muon step on a GPU with NCCL and the library (needs a B200).

The step's collectives (reduce-scatter of the gradients, all-gather of the
weights) run on a one-rank NCCL group, so the whole multi-GPU code path runs
-- flat buffers, bucketed collectives, the library's fused step on each
bucket's views -- on the one GPU available; the exchange between ranks itself
is covered on CPU by tests/test_shard_gloo.py.  A 2-layer slice of the 7B set
(CMuon-split QKV included) at T = 128, compared with the fp64 oracle on
sampled tiles: M' within one bf16 ulp, O within 3e-2 per tile and singular
values within 0.05, W' = W - lr O within bf16 rounding.
"""
import os
import socket

import numpy as np
import pytest

import oracle
from tests.parity_util import bf16_ulp
from tiled_newton_schulz_b200 import inputs, shard

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

C32 = [tuple(float(np.float32(v)) for v in inputs.QUINTIC)] * 5
MU, LR = 0.95, 0.02


@pytest.fixture(scope="module")
def hm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_newton_schulz_b200 import himuon
    himuon.load()
    return himuon


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def f64(t):
    return t.detach().double().cpu().numpy()


def test_flat_sharded_step_nccl_one_rank(hm):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120))
    try:
        wl = inputs.llama7b_set(2)
        shapes = [(m.rows, m.cols) for m in wl.matrices]
        splits = [m.split for m in wl.matrices]
        fs = shard.FlatShards(shapes, splits, 128, 1, buckets=3)
        W_flat = torch.empty(fs.total, dtype=torch.bfloat16, device=dev)
        G_flat = torch.empty_like(W_flat)
        O_flat = torch.zeros_like(W_flat)
        M_mine = torch.empty(fs.mine_total, dtype=torch.bfloat16, device=dev)
        Wv, Gv, Ov, Mv = fs.views(W_flat), fs.views(G_flat), fs.views(O_flat), fs.mine_views(M_mine, 0)
        for i, (H, W) in enumerate(shapes):
            Wv[i].copy_(inputs.gaussian_torch(H, W, 3 * i, dev, torch.float32) * 0.02)
            Mv[i].copy_(inputs.low_rank_plus_noise_torch(H, W, 64, 0.01, 3 * i + 1, dev))
            Gv[i].copy_(inputs.low_rank_plus_noise_torch(H, W, 64, 0.01, 3 * i + 2, dev))
        rng = np.random.default_rng(3)
        picks = []
        for _ in range(16):
            i = int(rng.integers(len(shapes)))
            H, W = shapes[i]
            r0, c0 = 128 * int(rng.integers(H // 128)), 128 * int(rng.integers(W // 128))
            picks.append((i, r0, c0))
        before = [(f64(Wv[i][r:r + 128, c:c + 128]), f64(Mv[i][r:r + 128, c:c + 128]), f64(Gv[i][r:r + 128, c:c + 128]))
                  for (i, r, c) in picks]
        p = hm.params(128, inputs.QUINTIC, steps=5)
        shard.flat_sharded_step(W_flat, G_flat, M_mine, fs, MU, LR, p, O_flat=O_flat)
        torch.cuda.synchronize()
        assert hm.device_status() == 0
        lr32 = float(np.float32(LR))
        for (i, r, c), (w0, m0, g0) in zip(picks, before):
            W2, M2, O = oracle.momentum_step(w0, m0, g0, MU, LR, 128, C32)
            assert np.all(np.abs(f64(Mv[i][r:r + 128, c:c + 128]) - M2) <= bf16_ulp(M2))
            got = f64(Ov[i][r:r + 128, c:c + 128])
            assert np.linalg.norm(got - O) / np.linalg.norm(O) <= 3e-2
            sv = np.abs(np.linalg.svd(got, compute_uv=False) - np.linalg.svd(O, compute_uv=False)).max()
            assert sv <= 0.05
            # W' is W - lr O with the fp32 O behind the stored bf16 one, rounded once to
            # bf16: within one bf16 ulp of W' plus lr times one bf16 ulp of O
            wexp = w0 - lr32 * got
            bound = bf16_ulp(wexp) + lr32 * bf16_ulp(got) + 1e-12
            assert np.all(np.abs(f64(Wv[i][r:r + 128, c:c + 128]) - wexp) <= bound)
    finally:
        dist.destroy_process_group()
