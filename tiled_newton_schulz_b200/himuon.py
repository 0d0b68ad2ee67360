"""Thin ctypes binding of libhimuon (argument marshalling only).

Every step of the path runs in the library's CUDA kernels; this module only
turns torch tensors into ``himuon_mat`` records, passes the current CUDA
stream, and allocates the caller-side workspace with torch when the caller
does not pass one.  Importing works without a GPU; any compute call without
the built library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhimuon.so")

BF16, FP16, FP32 = 0, 1, 2
OK = 0
OP_NS_TILED, OP_NS_FULL, OP_GRAM_NS, OP_MOMENTUM_STEP = 0, 1, 2, 3
EXPORTS = ("himuon_ns_tiled", "himuon_ns_full", "himuon_gram_ns", "himuon_momentum_step",
           "himuon_workspace_size", "himuon_get_device_status", "himuon_status_string",
           "himuon_version", "himuon_plan_tiles", "himuon_launch_count", "himuon_ns_static")
ERR_TOO_LARGE = -9
STATIC_SCRATCH_BYTES = 32 << 20


class Mat(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("ld", ctypes.c_int64), ("dtype", ctypes.c_int32)]


class Split(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int32), ("nblocks", ctypes.c_int32), ("sizes", ctypes.POINTER(ctypes.c_int64))]


class Params(ctypes.Structure):
    _fields_ = [("tile", ctypes.c_int32), ("steps", ctypes.c_int32), ("coeffs", ctypes.POINTER(ctypes.c_float)),
                ("eps", ctypes.c_float), ("compute", ctypes.c_int32), ("safety", ctypes.c_float),
                ("n_restart", ctypes.c_int32), ("restart_at", ctypes.POINTER(ctypes.c_int32)),
                ("chunk_bytes", ctypes.c_int64), ("tiles", ctypes.POINTER(ctypes.c_int32))]


class HimuonError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


_lib = None


def load() -> ctypes.CDLL:
    """Load the in-tree libhimuon.so; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m tiled_newton_schulz_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, vp, i32, i64 = ctypes.POINTER, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        ns_sig = [P(Mat), P(Mat), i32, P(Split), P(Params), vp, ctypes.c_size_t, vp]
        for name in ("himuon_ns_tiled", "himuon_ns_full", "himuon_gram_ns"):
            getattr(lib, name).argtypes = ns_sig
            getattr(lib, name).restype = ctypes.c_int
        lib.himuon_ns_static.argtypes = [P(Mat), P(Mat), i32, P(Split), P(Params), vp]
        lib.himuon_ns_static.restype = ctypes.c_int
        lib.himuon_momentum_step.argtypes = [P(Mat), P(Mat), P(Mat), i32, ctypes.c_float, ctypes.c_float, P(Split),
                                             P(Params), P(Mat), vp, ctypes.c_size_t, vp]
        lib.himuon_momentum_step.restype = ctypes.c_int
        lib.himuon_workspace_size.argtypes = [P(Mat), i32, P(Split), P(Params), i32]
        lib.himuon_workspace_size.restype = i64
        lib.himuon_get_device_status.argtypes = [vp]
        lib.himuon_get_device_status.restype = ctypes.c_int
        lib.himuon_status_string.argtypes = [ctypes.c_int]
        lib.himuon_status_string.restype = ctypes.c_char_p
        lib.himuon_version.restype = ctypes.c_int
        lib.himuon_launch_count.restype = i64
        lib.himuon_plan_tiles.argtypes = [P(Mat), i32, P(Split), i32, P(i64), i64]
        lib.himuon_plan_tiles.restype = i64
        _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load().himuon_status_string(int(code)).decode()


def _check(code: int, what: str) -> None:
    if code != OK:
        raise HimuonError(code, what)


# ---------------------------------------------------------------- marshalling

def _dtype_code(t) -> int:
    import torch
    return {torch.bfloat16: BF16, torch.float16: FP16, torch.float32: FP32}[t.dtype]


def mat(t) -> Mat:
    """himuon_mat of a 2-D tensor whose rows are contiguous (stride(1) == 1)."""
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("himuon needs 2-D tensors with unit column stride")
    return Mat(t.data_ptr(), t.shape[0], t.shape[1], t.stride(0), _dtype_code(t))


def _mats(ts) -> ctypes.Array:
    arr = (Mat * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = mat(t)
    return arr


def _splits(splits, n):
    """splits: None or a list of n entries, each None or (dim, sizes)."""
    if splits is None:
        return None, []
    arr = (Split * n)()
    keep = []
    for i, s in enumerate(splits):
        if s is None:
            arr[i] = Split(0, 0, None)
            continue
        dim, sizes = s
        sz = (ctypes.c_int64 * len(sizes))(*sizes)
        keep.append(sz)
        arr[i] = Split(int(dim), len(sizes), ctypes.cast(sz, ctypes.POINTER(ctypes.c_int64)))
    return arr, keep


def params(tile: int, coeffs, steps: int | None = None, eps: float = 1e-7, compute: int = BF16,
           safety: float = 1.0, restart: Sequence[int] = (), chunk_bytes: int = 0,
           tiles: Sequence[int] | None = None):
    """himuon_ns_params.  `tiles`: None, or one T per matrix of the call (it
    then replaces `tile`; T <= 0 is the whole matrix), e.g. the output of a
    runtime tile-size schedule (``schedule.TileSchedule``, ``schedule.choose_tiles``)."""
    flat = [float(v) for tri in (coeffs if isinstance(coeffs[0], (list, tuple)) else [coeffs]) for v in tri]
    if steps is not None and len(flat) == 3:
        flat = flat * steps
    K = len(flat) // 3
    c = (ctypes.c_float * len(flat))(*flat)
    r = (ctypes.c_int32 * max(1, len(restart)))(*restart)
    p = Params(int(tile), K, ctypes.cast(c, ctypes.POINTER(ctypes.c_float)), float(eps), int(compute), float(safety),
               len(restart), ctypes.cast(r, ctypes.POINTER(ctypes.c_int32)), int(chunk_bytes), None)
    tl = None
    if tiles is not None:
        tl = (ctypes.c_int32 * max(1, len(tiles)))(*[int(t) for t in tiles])
        p.tiles = ctypes.cast(tl, ctypes.POINTER(ctypes.c_int32))
    p._keep = (c, r, tl)
    p._ntiles = None if tiles is None else len(tiles)
    return p


def _check_tiles(p: Params, n: int) -> None:
    """The library reads one tile size per matrix from p.tiles: the list must
    have exactly n entries (the C side cannot see its length)."""
    if _has_tiles(p) and getattr(p, "_ntiles", None) != n:
        raise ValueError(f"params.tiles has {getattr(p, '_ntiles', '?')} entries for {n} matrices")


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(tensors, p: Params, op: int, splits=None) -> int:
    _check_tiles(p, len(tensors))
    m = _mats(tensors)
    sp, _keep = _splits(splits, len(tensors))
    n = load().himuon_workspace_size(m, len(tensors), sp, ctypes.byref(p), op)
    if n < 0:
        raise HimuonError(int(n), "himuon_workspace_size")
    return int(n)


def _workspace(tensors, p, op, splits, workspace):
    import torch
    if workspace is not None:
        return workspace.data_ptr(), workspace.numel() * workspace.element_size(), workspace
    need = workspace_size(tensors, p, op, splits)
    if need == 0:
        return None, 0, None
    ws = torch.empty(need, dtype=torch.uint8, device=tensors[0].device)
    return ws.data_ptr(), need, ws


def _ns_call(fn_name, op, inputs, outputs, p, splits, workspace, stream):
    if len(inputs) != len(outputs):
        raise ValueError("inputs and outputs differ in length")
    _check_tiles(p, len(inputs))
    mi, mo = _mats(inputs), _mats(outputs)
    sp, _keep = _splits(splits, len(inputs))
    wp, wb, _ws = _workspace(inputs, p, op, splits, workspace)
    rc = getattr(load(), fn_name)(mi, mo, len(inputs), sp, ctypes.byref(p), wp, wb, _stream(stream))
    _check(rc, fn_name)
    return _ws


def _has_tiles(p: Params) -> bool:
    return bool(ctypes.cast(p.tiles, ctypes.c_void_p).value)


def ns_tiled(inputs, outputs, p: Params, splits=None, workspace=None, stream=None):
    op = OP_NS_TILED if (_has_tiles(p) or p.tile > 0) else OP_NS_FULL
    return _ns_call("himuon_ns_tiled", op, inputs, outputs, p, splits, workspace, stream)


def ns_full(inputs, outputs, p: Params, splits=None, workspace=None, stream=None):
    return _ns_call("himuon_ns_full", OP_NS_FULL, inputs, outputs, p, splits, workspace, stream)


def gram_ns(inputs, outputs, p: Params, splits=None, workspace=None, stream=None):
    return _ns_call("himuon_gram_ns", OP_GRAM_NS, inputs, outputs, p, splits, workspace, stream)


def ns_static(inputs, outputs, p: Params, splits=None, stream=None) -> int:
    """Staged NS with the library's own fixed device scratch (no workspace).

    For callers that cannot allocate device memory; returns the status code
    (ERR_TOO_LARGE when the call does not fit the 32 MiB array) instead of
    raising, so callers can fall back.
    """
    if len(inputs) != len(outputs):
        raise ValueError("inputs and outputs differ in length")
    mi, mo = _mats(inputs), _mats(outputs)
    sp, _keep = _splits(splits, len(inputs))
    return int(load().himuon_ns_static(mi, mo, len(inputs), sp, ctypes.byref(p), _stream(stream)))


def momentum_step(W, M, G, mu: float, lr: float, p: Params, splits=None, update_out=None, workspace=None,
                  stream=None):
    """M <- mu M + G; O = tiledNS(M); W <- W - lr O (W may be None); O to update_out."""
    n = len(M)
    _check_tiles(p, n)
    mw = _mats(W) if W is not None else None
    mm, mg = _mats(M), _mats(G)
    mo = _mats(update_out) if update_out is not None else None
    sp, _keep = _splits(splits, n)
    wp, wb, _ws = _workspace(M, p, OP_MOMENTUM_STEP, splits, workspace)
    rc = load().himuon_momentum_step(mw, mm, mg, n, float(mu), float(lr), sp, ctypes.byref(p), mo, wp, wb,
                                     _stream(stream))
    _check(rc, "himuon_momentum_step")
    return _ws


def launch_count() -> int:
    """Kernels the library has enqueued since it was loaded (host counter)."""
    return int(load().himuon_launch_count())


def device_status(stream=None) -> int:
    return int(load().himuon_get_device_status(_stream(stream)))


def plan_tiles(shapes, splits=None, tile: int = 128):
    """Tile list the scheduler numbers, as (matrix, row0, col0, h, w) tuples.

    Host-only: the matrices are described by shape alone (a dummy pointer).
    """
    n = len(shapes)
    arr = (Mat * n)()
    for i, (r, c) in enumerate(shapes):
        arr[i] = Mat(0x1000, r, c, c, BF16)
    sp, _keep = _splits(splits, n)
    lib = load()
    total = lib.himuon_plan_tiles(arr, n, sp, int(tile), None, 0)
    if total < 0:
        raise HimuonError(int(total), "himuon_plan_tiles")
    rec = (ctypes.c_int64 * (5 * max(1, total)))()
    lib.himuon_plan_tiles(arr, n, sp, int(tile), rec, total)
    return [tuple(rec[5 * i:5 * i + 5]) for i in range(total)]
