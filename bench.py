"""Throughput of the tiled-NS optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--tile 128] [--impl ours|reference]

Workload (default): one full Muon step over every 2-D weight of a Llama-style
7B shape (32 layers; fused QKV 4096x12288 split into three 4096x4096 blocks;
O 4096x4096; gate/up 4096x11008; down 11008x4096): M <- 0.95 M + G,
O = tiledNS_T(M) with K = 5 quintic steps, W <- W - 0.02 O, all bf16 in HBM
(38.9 GB of W, M, G).  Synthetic inputs: M and G low-rank-plus-noise
(U diag(1/i) V^T, rank 64, Haar U, V, + 0.01 N(0,1)), W = 0.02 N(0,1).

A step is one himuon_momentum_step call over all matrices.  The inputs
(38.9 GB) are far larger than L2 (126 MB), so no flush is needed between
steps.  Time is taken with CUDA events on the launching stream.

With N > 1 (under torchrun, one rank per GPU, NCCL) the step is the
data-parallel sharded step of ``shard.flat_sharded_step``: every rank holds
the replicated weights and its own gradients for the whole 7B set in flat
buffers, the gradients are reduce-scattered (averaged) onto the owners of the
matrices, each rank runs the fused library step on its own matrices (the
momentum lives only there), and the weights are all-gathered, in buckets that
overlap the collectives with the steps.  The job processes the 7B set once
per step (strong scaling); the max over ranks is reported.  ``--sharded``
runs the same code path on one rank.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

QUINTIC = (3.4445, -4.7750, 2.0315)
K_STEPS = 5
AUTO_CANDIDATES = (128, 256, 512, 0)    # T = 32 / 64 cost more than 128 on chip and couple less
MU, LR = 0.95, 0.02
METRIC = "tiled-NS step: matrix elements/s"


# ---------------------------------------------------------------- helpers

def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def flops_per_tile(h: int, w: int, K: int) -> float:
    """The pages' per-step count 2(2 alpha + 1) n^3 for an n x m tile, n <= m."""
    n, m = min(h, w), max(h, w)
    return K * (4.0 * m * n * n + 2.0 * n ** 3)


def sym_flops_per_tile(h: int, w: int, K: int) -> float:
    """The symmetric-minimal count (3 alpha + 1) n^3 per step: X X^T and A^2
    credited as their triangles (half of 2 m n^2 and of 2 n^3), B X in full."""
    n, m = min(h, w), max(h, w)
    return K * (3.0 * m * n * n + 1.0 * n ** 3)


def workload_tiles(shapes_splits, T, sym=False):
    tiles, flops = 0, 0.0
    for (H, W), split in shapes_splits:
        blocks = [(H, W)] if split is None else [((H, s) if split[0] == 1 else (s, W)) for s in split[1]]
        for (h, w) in blocks:
            Tb = T if T > 0 else max(h, w)   # T <= 0: the whole block is one tile
            for r0 in range(0, h, Tb):
                for c0 in range(0, w, Tb):
                    th, tw = min(Tb, h - r0), min(Tb, w - c0)
                    tiles += 1
                    flops += (sym_flops_per_tile if sym else flops_per_tile)(th, tw, K_STEPS)
    return tiles, flops


class ClockSampler:
    """nvidia-smi clocks and throttle reasons while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        loaded = [s for s in sm if mx and s > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- workload

def llama7b_matrices(layers: int = 32):
    from tiled_newton_schulz_b200.inputs import llama7b_set
    wl = llama7b_set(layers)
    return [((m.rows, m.cols), m.split) for m in wl.matrices]


def make_state(device, seed_base: int, layers: int = 32):
    import torch
    from tiled_newton_schulz_b200.inputs import gaussian_torch, low_rank_plus_noise_torch
    mats = llama7b_matrices(layers)
    W, M, G = [], [], []
    for i, ((H, Wd), _) in enumerate(mats):
        W.append((gaussian_torch(H, Wd, seed_base + 3 * i, device, torch.float32) * 0.02).to(torch.bfloat16))
        M.append(low_rank_plus_noise_torch(H, Wd, 64, 0.01, seed_base + 3 * i + 1, device))
        G.append(low_rank_plus_noise_torch(H, Wd, 64, 0.01, seed_base + 3 * i + 2, device))
    torch.cuda.synchronize(device)
    return mats, W, M, G


def cpu_oracle_sample(mats_state, T: int, budget_s: float):
    """Oracle on tiles of layer 0 (strips of whole tiles) until the budget is used.

    Returns (elements/s, elements, seconds, threads, description)."""
    import numpy as np
    import oracle
    oracle.build()
    W, M, G = mats_state
    H, Wd = W.shape
    cols = 16 * T            # one strip of 16 tiles per call (OpenMP over its tiles)
    elems, t0, strips = 0, time.perf_counter(), 0
    while True:
        c0 = (strips % 2) * (Wd - cols)
        sl = np.s_[0:T, c0:c0 + cols]
        oracle.momentum_step(W[sl], M[sl], G[sl], MU, LR, T, [QUINTIC] * K_STEPS)
        elems += T * cols
        strips += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    desc = (f"{strips} strips of 16 {T}x{T} tiles from layer 0's O projection (fused momentum, "
            f"K={K_STEPS} NS steps, weight update), fp64")
    return elems / dt, elems, dt, oracle.num_threads(), desc


# ---------------------------------------------------------------- arms

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    rng = np.random.default_rng(5)
    T = args.tile
    H, Wd = 4096, 4096
    from tiled_newton_schulz_b200 import inputs
    W = 0.02 * rng.standard_normal((T, 16 * T))
    Mx = inputs.low_rank_plus_noise(T, 16 * T, inputs.sigma_inverse(64), 0.01, seed=1)
    Gx = inputs.low_rank_plus_noise(T, 16 * T, inputs.sigma_inverse(64), 0.01, seed=2)
    import oracle
    oracle.build()
    per_step = []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.momentum_step(W, Mx, Gx, MU, LR, T, [QUINTIC] * K_STEPS)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            per_step.append(dt)
    elems = T * 16 * T
    total = sum(per_step)
    value = elems * len(per_step) / total
    mats = llama7b_matrices()
    desc = (f"one strip of 16 {T}x{T} tiles per step (fused momentum, K={K_STEPS} NS steps, weight update) "
            f"of the Llama-7B step workload, fp64, low-rank-plus-noise inputs")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"llama7b_32l_full_step_T{T}", "tile": T, "steps_K": K_STEPS,
                   "matrices": len(mats), "sample_per_step_elements": elems},
        "cpu_baseline": {"value": value, "unit": "elements/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "elements/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_sharded(args):
    """The data-parallel sharded step (N ranks, NCCL) on the 7B set."""
    import datetime
    import torch
    import torch.distributed as dist
    from tiled_newton_schulz_b200 import himuon as hm
    from tiled_newton_schulz_b200 import shard
    from tiled_newton_schulz_b200.inputs import gaussian_torch, low_rank_plus_noise_torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world == 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29511")
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    hm.load()
    T = args.tile
    compute = {"bf16": hm.BF16, "fp16": hm.FP16}[args.compute]
    mats = llama7b_matrices(args.layers)
    shapes, splits = [s for s, _ in mats], [sp for _, sp in mats]
    elements = sum(H * Wd for H, Wd in shapes)
    n_tiles, flops = workload_tiles(mats, T)
    fs = shard.FlatShards(shapes, splits, T, world, buckets=args.buckets)
    W_flat = torch.empty(fs.total, dtype=torch.bfloat16, device=device)
    G_flat = torch.empty_like(W_flat)
    M_mine = torch.empty(fs.mine_total, dtype=torch.bfloat16, device=device)
    Wv, Gv, Mv = fs.views(W_flat), fs.views(G_flat), fs.mine_views(M_mine, rank)
    for i, (H, Wd) in enumerate(shapes):
        # the same weights on every rank, this rank's own gradients, momentum on the owner
        Wv[i].copy_(gaussian_torch(H, Wd, 3 * i, device, torch.float32) * 0.02)
        Gv[i].copy_(low_rank_plus_noise_torch(H, Wd, 64, 0.01, 1000 * rank + 3 * i + 2, device))
        if Mv[i] is not None:
            Mv[i].copy_(low_rank_plus_noise_torch(H, Wd, 64, 0.01, 3 * i + 1, device))
    torch.cuda.synchronize(device)
    p = hm.params(T, QUINTIC, steps=K_STEPS, compute=compute)
    stream = torch.cuda.current_stream(device)

    def step():
        shard.flat_sharded_step(W_flat, G_flat, M_mine, fs, MU, LR, p)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    st = hm.device_status()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    dist.barrier()
    torch.cuda.synchronize(device)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    launches0 = hm.launch_count()
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    launches = hm.launch_count() - launches0
    torch.cuda.synchronize(device)
    dist.barrier()
    clk = clocks.stop()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    t = torch.tensor([evs[0].elapsed_time(evs[-1])] + per + [float(st != 0)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms, per, bad = float(t[0].item()), [float(v) for v in t[1:-1].tolist()], t[-1].item() > 0
    ms_step = ms / args.steps
    peaks, peak_src = read_peaks()
    peak_burst = float(peaks.get("bf16_tflops"))
    achieved = flops / (ms_step / 1e3) / 1e12
    bytes_coll = 2 * 2.0 * elements * (world - 1) / world   # bf16 reduce-scatter of G + all-gather of W, per rank
    line = {
        "metric": METRIC, "value": elements / (ms_step / 1e3), "unit": "elements/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": args.compute, "data": "synthetic",
        "config": {"workload": f"llama7b_{args.layers}l_full_step_T{T}", "tile": T, "steps_K": K_STEPS, "mu": MU,
                   "lr": LR, "matrices": len(mats), "tiles": n_tiles, "elements_total": elements,
                   "storage": "bf16 W, M, G", "accumulate": "fp32",
                   "l2": f"inputs {6 * elements / 1e9:.1f} GB >> 126 MB L2, no flush",
                   "parallelism": (f"dp{world}: gradients reduce-scattered onto matrix owners, fused step on own "
                                   f"matrices, weights all-gathered (NCCL), {fs.buckets} buckets"),
                   "flop_imbalance": fs.imbalance(T)},
        "ms_per_step_median": statistics.median(per), "ms_per_step_min": min(per),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_burst * world, "unit": "TFLOP/s",
                     "frac": achieved / (peak_burst * world), "traffic": None,
                     "peak_source": f"bf16_tflops x {world} GPUs ({peak_src})",
                     "collective_bytes_per_rank": bytes_coll,
                     "collective_time_ms_at_770GBps": bytes_coll / 770e9 * 1e3},
        "cpu_baseline": None,
        "e2e": {"value": None, "unit": "elements/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0,
                "note": "not measured for the sharded step: the whole gradient of every rank would cross PCIe"},
        "gpu_launches": launches, "clocks": clk, "device_status_ok": not bad,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    from tiled_newton_schulz_b200 import himuon as hm

    # one GPU (N > 1 runs the sharded step, run_sharded)
    world, rank, local = 1, 0, int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    hm.load()

    T = args.tile
    compute = {"bf16": hm.BF16, "fp16": hm.FP16}[args.compute]
    mats, W, M, G = make_state(device, seed_base=1000 * rank, layers=args.layers)
    splits = [s for (_, s) in mats]
    elements = sum(H * Wd for (H, Wd), _ in mats)
    tiles = None
    if args.budget_ms is not None:
        # runtime tile-size choice: per matrix, the largest T whose measured
        # step cost keeps the set within the budget (untimed, before warm-up)
        from tiled_newton_schulz_b200 import schedule
        costs = schedule.measure_costs([s for s, _ in mats], splits, candidates=AUTO_CANDIDATES, compute=compute,
                                       reps=2, device=device, op="step")
        tiles = schedule.choose_tiles(costs, args.budget_ms / 1e3)
        modeled_ms = schedule.modeled_cost(costs, tiles) * 1e3
        n_tiles, flops = 0, 0.0
        for m, t in zip(mats, tiles):
            a, b = workload_tiles([m], t if t > 0 else 1 << 30)
            n_tiles, flops = n_tiles + a, flops + b
    else:
        n_tiles, flops = workload_tiles(mats, T)
    p = hm.params(T, QUINTIC, steps=K_STEPS, compute=compute, tiles=tiles)
    ws_need = hm.workspace_size(M, p, hm.OP_MOMENTUM_STEP, splits)
    ws = torch.empty(max(ws_need, 256), dtype=torch.uint8, device=device) if ws_need else None
    stream = torch.cuda.current_stream(device)

    def step():
        hm.momentum_step(W, M, G, MU, LR, p, splits=splits, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    st = hm.device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {hm.status_string(st)}")

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    torch.cuda.synchronize(device)
    # one event between consecutive steps: the whole region and every step's time
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    launches0 = hm.launch_count()
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    launches = hm.launch_count() - launches0
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    ms = evs[0].elapsed_time(evs[-1])
    per_step_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    st = hm.device_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {hm.status_string(st)}")
    ms_step = ms / args.steps
    value = world * elements / (ms_step / 1e3)
    tflops = world * flops / (ms_step / 1e3) / 1e12

    # end to end through the public API with host buffers (pinned), this rank's replica
    e2e_value, h2d, d2h = None, 0, 0
    if not args.no_e2e:
        hW = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in W]
        hM = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in M]
        hG = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in G]
        for h, d in zip(hW + hM + hG, W + M + G):
            h.copy_(d)
        h2d = sum(x.numel() * x.element_size() for x in hW + hM + hG)
        d2h = sum(x.numel() * x.element_size() for x in hW + hM)
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        # The step in chunks of whole layers on three streams: a chunk's upload,
        # the previous chunk's NS step and the download of the one before run
        # at once (PCIe carries both directions concurrently).  Each chunk is
        # one public-API call on its own stream; at most 16 chunks, so their
        # plans stay cached.
        n_mat = len(mats)
        per = max(1, -(-n_mat // 16))
        per = -(-per // 5) * 5 if n_mat % 5 == 0 else per     # whole layers (5 matrices each)
        chunks = [list(range(i, min(n_mat, i + per))) for i in range(0, n_mat, per)]
        p_chunk = [p if tiles is None else hm.params(T, QUINTIC, steps=K_STEPS, compute=compute,
                                                     tiles=[tiles[i] for i in idx]) for idx in chunks]
        s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))

        def e2e_step():
            start = torch.cuda.Event()
            start.record(stream)
            for s in (s_in, s_cmp, s_out):
                s.wait_event(start)
            done_out = None
            for idx, pc in zip(chunks, p_chunk):
                with torch.cuda.stream(s_in):
                    for i in idx:
                        W[i].copy_(hW[i], non_blocking=True)
                        M[i].copy_(hM[i], non_blocking=True)
                        G[i].copy_(hG[i], non_blocking=True)
                    e_in = torch.cuda.Event()
                    e_in.record(s_in)
                s_cmp.wait_event(e_in)
                hm.momentum_step([W[i] for i in idx], [M[i] for i in idx], [G[i] for i in idx], MU, LR, pc,
                                 splits=[splits[i] for i in idx], workspace=ws, stream=s_cmp)
                e_c = torch.cuda.Event()
                e_c.record(s_cmp)
                s_out.wait_event(e_c)
                with torch.cuda.stream(s_out):
                    for i in idx:
                        hW[i].copy_(W[i], non_blocking=True)
                        hM[i].copy_(M[i], non_blocking=True)
                    done_out = torch.cuda.Event()
                    done_out.record(s_out)
            stream.wait_event(done_out)

        e2e_step()
        torch.cuda.synchronize(device)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize(device)
        ems = a0.elapsed_time(a1)
        e2e_value = world * elements / (ems / e2e_steps / 1e3)
        del hW, hM, hG

    # CPU baseline: the oracle on a bounded sample, rank 0 at N = 1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and tiles is None:
        idx = 1  # layer 0, O projection (4096 x 4096)
        sample = tuple(x[idx][:T].detach().double().cpu().numpy() for x in (W, M, G))
        v, e, dt, threads, desc = cpu_oracle_sample(sample, T, args.cpu_budget)
        cpu = {"value": v, "unit": "elements/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": round(dt, 2)}

    peaks, peak_src = read_peaks()
    peak_sus = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    peak_burst = float(peaks.get("bf16_tflops"))
    hbm = float(peaks.get("hbm_gbs"))
    # the step is a single launch of the on-chip kernel: launch duration = step time
    # (with per-matrix tile sizes it is several launches; the figure is then the step's).
    # The launch takes tens of ms and runs alone: the burst peak is its denominator;
    # the sustained one (a seconds-long GEMM loop under the power cap) is given beside it.
    achieved = flops / (ms_step / 1e3) / 1e12
    if tiles is None:
        _, sym_flops = workload_tiles(mats, T, sym=True)
    else:
        sym_flops = sum(workload_tiles([m], t if t > 0 else 1 << 30, sym=True)[1] for m, t in zip(mats, tiles))
    bytes_step = 10 * elements
    t_roof = max(flops / (peak_burst * 1e12), bytes_step / (hbm * 1e9))
    t_roof_sym = max(sym_flops / (peak_burst * 1e12), bytes_step / (hbm * 1e9))
    prof = load_profile_traffic(T) if tiles is None else None
    roofline = {
        "bound": "tensor", "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s", "frac": achieved / peak_burst,
        "traffic": prof,
        "kernel": ((ONCHIP_KERNELS[T] + "_kernel" if T in ONCHIP_KERNELS else "gemm_tc_kernel (staged path)")
                   if tiles is None else "whole step (on-chip and staged launches)"),
        "peak_source": f"bf16_tflops, burst ({peak_src})",
        "frac_sustained": achieved / peak_sus, "peak_sustained": peak_sus,
        "frac_sym": sym_flops / (ms_step / 1e3) / 1e12 / peak_burst,
        "achieved_sym": sym_flops / (ms_step / 1e3) / 1e12,
        "frac_of_roofline_time": t_roof / (ms_step / 1e3), "frac_of_roofline_time_sym": t_roof_sym / (ms_step / 1e3),
        "flops_per_launch": flops, "flop_count": "nominal: 2(2a+1)n^3 per NS step per tile (a = m/n)",
        "sym_flops_per_launch": sym_flops, "sym_flop_count": "(3a+1)n^3 per NS step per tile (triangles of X X^T, A^2)",
        "hbm_bytes_per_launch": bytes_step, "hbm_time_ms": bytes_step / (hbm * 1e9) * 1e3,
        "tensor_time_ms_burst_peak": flops / (peak_burst * 1e12) * 1e3,
    }
    line = {
        "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": args.compute, "data": "synthetic",
        "config": {"workload": (f"llama7b_{args.layers}l_full_step_T{T}" if tiles is None else
                                f"llama7b_{args.layers}l_full_step_autoT_budget{args.budget_ms:g}ms"),
                   "tile": T if tiles is None else "per matrix", "steps_K": K_STEPS, "mu": MU, "lr": LR,
                   "matrices": len(mats), "split_blocks": sum(len(s[1]) if s else 1 for s in splits),
                   "tiles": n_tiles, "elements_per_gpu": elements, "storage": "bf16 W, M, G",
                   "accumulate": "fp32",
                   "l2": f"inputs {6 * elements / 1e9:.1f} GB per GPU >> 126 MB L2, no flush",
                   "parallelism": "one GPU"},
        "tflops": tflops,
        "ms_per_step_median": statistics.median(per_step_ms), "ms_per_step_min": min(per_step_ms),
        "ms_per_step_max": max(per_step_ms),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "elements/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if tiles is not None:
        mix = {}
        for t in tiles:
            mix[str(t if t > 0 else "whole")] = mix.get(str(t if t > 0 else "whole"), 0) + 1
        line["config"].update({"tile_mix": mix, "candidates": list(AUTO_CANDIDATES), "budget_ms": args.budget_ms,
                               "modeled_ms": modeled_ms,
                               "cost_model": "momentum_step per matrix at each T, CUDA events, batched per shape"})
    print(json.dumps(line), flush=True)
    return 0


ONCHIP_KERNELS = {128: "ns_resident", 256: "ns_pair"}   # the on-chip kernel of each tile edge
KERNEL_HEADERS = ("onchip.cuh", "ptx.cuh")


def kernel_source_sha(kernel: str) -> str:
    """sha256 prefix of an on-chip kernel's source and the device headers it shares."""
    import hashlib
    h = hashlib.sha256()
    for name in (kernel + ".cu",) + KERNEL_HEADERS:
        with open(os.path.join(ROOT, "tiled_newton_schulz_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_profile_traffic(T: int):
    """DRAM bytes per launch of the on-chip kernel from the committed ncu
    summary, or None when there is none or the kernel source changed since."""
    kernel = ONCHIP_KERNELS.get(T)
    if kernel is None:
        return None
    p = os.path.join(ROOT, "profiles", f"{kernel}_llama7b_T{T}_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        sha = kernel_source_sha(kernel)
    except OSError:
        return None
    return d.get("dram_bytes_per_full_launch") if d.get("kernel_source_sha256_prefix") == sha else None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--tile", type=int, default=128)
    ap.add_argument("--layers", type=int, default=32, help="transformer layers of the 7B shape set")
    ap.add_argument("--compute", choices=["bf16", "fp16"], default="bf16")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--sharded", action="store_true", help="time the data-parallel sharded step even on one rank")
    ap.add_argument("--buckets", type=int, default=4, help="buckets of the sharded step's collectives")
    ap.add_argument("--budget-ms", type=float, default=None,
                    help="choose T per matrix at run time: the largest tiles whose measured cost fits this budget")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 or args.sharded:
        return run_sharded(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
