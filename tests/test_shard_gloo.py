"""Multi-rank path on CPU (gloo, world_size 2): matrices are assigned to ranks
by FLOPs, each rank runs the fp64 oracle on its own matrices, the results are
gathered, and rank 0 checks they equal the single-process result bit for bit
and that every matrix was processed exactly once."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from tiled_newton_schulz_b200 import inputs, shard

SHAPES = [(64, 96), (40, 72), (96, 32), (48, 48), (16, 80)]
SPLITS = [None, (1, (24, 48)), None, (0, (16, 32)), None]
T = 16


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = shard.assign_matrices(SHAPES, SPLITS, T, world)[rank]
        res = {}
        for i in mine:
            X = inputs.gaussian(SHAPES[i], seed=100 + i)
            res[i] = oracle.ns_tiled_split(X, T, [inputs.QUINTIC] * 5, split=SPLITS[i])
        gathered = [None] * world
        dist.all_gather_object(gathered, res)
        if rank == 0:
            merged, counts = {}, {}
            for part in gathered:
                for i, v in part.items():
                    counts[i] = counts.get(i, 0) + 1
                    merged[i] = v
            ok = sorted(counts) == list(range(len(SHAPES))) and all(c == 1 for c in counts.values())
            for i in range(len(SHAPES)):
                X = inputs.gaussian(SHAPES[i], seed=100 + i)
                ref = oracle.ns_tiled_split(X, T, [inputs.QUINTIC] * 5, split=SPLITS[i])
                ok = ok and np.array_equal(merged[i], ref)
            q.put(ok)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_tiled_ns_matches_single_process():
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    assert q.get(timeout=10) is True


def test_assignment_covers_each_matrix_once_and_balances():
    wl = inputs.llama7b_set(32)
    shapes = [(m.rows, m.cols) for m in wl.matrices]
    splits = [m.split for m in wl.matrices]
    for world in (1, 2, 4, 8):
        a = shard.assign_matrices(shapes, splits, 128, world)
        flat = sorted(i for lst in a for i in lst)
        assert flat == list(range(len(shapes)))
        assert shard.imbalance(shapes, splits, 128, a) < 1.05
