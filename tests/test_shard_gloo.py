"""Multi-rank path on CPU (gloo, world_size 2): matrices are assigned to ranks
by FLOPs, each rank runs the fp64 oracle on its own matrices, the results are
gathered, and rank 0 checks they equal the single-process result bit for bit
and that every matrix was processed exactly once.  The sharded Muon step
(gradients reduced onto owners, the owner's step, weights broadcast) runs with
the oracle as its step function and must equal the single-process step on the
averaged gradients; incomplete inputs on one rank make every rank raise."""
import os
import socket

import numpy as np
import pytest
import torch
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


MU, LR = 0.95, 0.02


def _oracle_step(T):
    """Step function with the library's signature, computed by the fp64 oracle
    in place on CPU tensors (the sharded step calls the library on a GPU)."""
    import oracle

    def step(W, M, G, mu, lr, p, splits=None):
        for k in range(len(W)):
            sp = None if splits is None else splits[k]
            mp = oracle.momentum(M[k].numpy(), G[k].numpy(), mu)
            O = oracle.ns_tiled_split(mp, T, [inputs.QUINTIC] * 5, split=sp)
            M[k].copy_(torch.from_numpy(mp))
            W[k].sub_(lr * torch.from_numpy(O))
    return step


def _state(rank):
    W = [torch.from_numpy(0.02 * inputs.gaussian(s, seed=200 + i)) for i, s in enumerate(SHAPES)]
    M = [torch.from_numpy(inputs.gaussian(s, seed=300 + i)) for i, s in enumerate(SHAPES)]
    G = [torch.from_numpy(inputs.gaussian(s, seed=400 + 10 * i + rank)) for i, s in enumerate(SHAPES)]
    return W, M, G


def _step_worker(rank, world, port, q, broken):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assignment = shard.assign_matrices(SHAPES, SPLITS, T, world)
        W, M, G = _state(rank)
        own = shard.owners(assignment, len(SHAPES))
        M = [m if own[i] == rank else None for i, m in enumerate(M)]
        if broken and rank == 1:
            M[assignment[1][0]] = None
        try:
            shard.sharded_momentum_step(W, M, G, MU, LR, None, assignment, splits=SPLITS, step_fn=_oracle_step(T))
        except ValueError as e:
            q.put((rank, "raised", str(e)))
            return
        q.put((rank, "done", [w.numpy() for w in W], {i: M[i].numpy() for i in assignment[rank]}))
    finally:
        dist.destroy_process_group()


def _run_step(broken):
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_step_worker, args=(r, 2, port, q, broken)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    return sorted(out, key=lambda r: r[0])


def test_two_rank_sharded_momentum_step_matches_single_process():
    import oracle
    out = _run_step(broken=False)
    assert [o[1] for o in out] == ["done", "done"]
    W, M, _ = _state(0)
    G = [(a + b) / 2 for a, b in zip(_state(0)[2], _state(1)[2])]
    for i in range(len(SHAPES)):
        mp = oracle.momentum(M[i].numpy(), G[i].numpy(), MU)
        Wr = W[i].numpy() - LR * oracle.ns_tiled_split(mp, T, [inputs.QUINTIC] * 5, split=SPLITS[i])
        for o in out:                       # every rank holds the same new weights
            assert np.array_equal(o[2][i], Wr), i
        owner = [o for o in out if i in o[3]]
        assert len(owner) == 1 and np.array_equal(owner[0][3][i], mp), i


def test_sharded_step_with_incomplete_inputs_raises_on_every_rank():
    out = _run_step(broken=True)
    assert [o[1] for o in out] == ["raised", "raised"]
    assert "rank 1 owns a matrix without momentum" in out[1][2]
    assert "another rank" in out[0][2]


def test_owners_rejects_bad_assignments():
    assert shard.owners([[0, 2], [1]], 3) == [0, 1, 0]
    with pytest.raises(ValueError):
        shard.owners([[0, 1], [1]], 3)
    with pytest.raises(ValueError):
        shard.owners([[0], [2]], 3)


# ---------------------------------------------------------------- flat buffers

def test_flat_placement_is_disjoint_aligned_and_bucketed():
    wl = inputs.llama7b_set(2)
    shapes = [(m.rows, m.cols) for m in wl.matrices]
    splits = [m.split for m in wl.matrices]
    for world in (1, 2, 3, 8):
        for buckets in (1, 2, 5):
            fs = shard.FlatShards(shapes, splits, 128, world, buckets=buckets)
            spans = sorted((o, o + h * w) for o, (h, w) in zip(fs.offset, shapes))
            assert all(a % 128 == 0 for a, _ in spans)
            assert all(b0 <= a1 for (_, b0), (a1, _) in zip(spans, spans[1:]))       # no overlap
            assert spans[-1][1] <= fs.total
            for i, (h, w) in enumerate(shapes):
                r, b = fs.owner[i], fs.bucket_of[i]
                lo = fs.bucket_base[b] + r * fs.slot_elems[b]
                assert lo <= fs.offset[i] and fs.offset[i] + h * w <= lo + fs.slot_elems[b]   # inside its slot
                mo = fs.mine_offset[i]
                assert 0 <= mo and mo + h * w <= fs.mine_total
            assert sorted(i for r in range(world) for b in range(fs.buckets) for i in fs.members[r][b]) == \
                list(range(len(shapes)))


def _flat_worker(rank, world, port, q, buckets, broken):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        fs = shard.FlatShards(SHAPES, SPLITS, T, world, buckets=buckets)
        W0, M0, G0 = _state(rank)
        W_flat = torch.zeros(fs.total, dtype=torch.float64)
        G_flat = torch.zeros(fs.total, dtype=torch.float64)
        M_mine = torch.zeros(fs.mine_total + (1 if broken and rank == 1 else 0), dtype=torch.float64)
        for v, x in zip(fs.views(W_flat), W0):
            v.copy_(x)
        for v, x in zip(fs.views(G_flat), G0):
            v.copy_(x)
        for i, v in enumerate(fs.mine_views(M_mine, rank)):
            if v is not None:
                v.copy_(M0[i])
        try:
            shard.flat_sharded_step(W_flat, G_flat, M_mine, fs, MU, LR, None, step_fn=_oracle_step(T))
        except ValueError as e:
            q.put((rank, "raised", str(e)))
            return
        mine = {i: v.numpy().copy() for i, v in enumerate(fs.mine_views(M_mine, rank)) if v is not None}
        q.put((rank, "done", [v.numpy().copy() for v in fs.views(W_flat)], mine))
    finally:
        dist.destroy_process_group()


def _run_flat(buckets, broken=False):
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_flat_worker, args=(r, 2, port, q, buckets, broken)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    return sorted(out, key=lambda r: r[0])


@pytest.mark.parametrize("buckets", [1, 3])
def test_two_rank_flat_sharded_step_matches_single_process(buckets):
    """Reduce-scatter of the gradients, each rank's step on its own matrices,
    all-gather of the weights: every rank ends with exactly the weights of a
    single-process step on the averaged gradients, and each owner with its
    matrices' new momentum."""
    import oracle
    out = _run_flat(buckets)
    assert [o[1] for o in out] == ["done", "done"]
    W, M, _ = _state(0)
    G = [(a + b) / 2 for a, b in zip(_state(0)[2], _state(1)[2])]
    for i in range(len(SHAPES)):
        mp_ = oracle.momentum(M[i].numpy(), G[i].numpy(), MU)
        Wr = W[i].numpy() - LR * oracle.ns_tiled_split(mp_, T, [inputs.QUINTIC] * 5, split=SPLITS[i])
        for o in out:
            assert np.array_equal(o[2][i], Wr), i
        owner = [o for o in out if i in o[3]]
        assert len(owner) == 1 and np.array_equal(owner[0][3][i], mp_), i


def test_flat_sharded_step_with_a_bad_buffer_raises_on_every_rank():
    out = _run_flat(2, broken=True)
    assert [o[1] for o in out] == ["raised", "raised"]
    assert "rank 1" in out[1][2] and "another rank" in out[0][2]
