"""Host-side checks of libhimuon (no GPU needed): the library loads, exports
every entry point the header declares, rejects bad arguments without touching
a device, and its tile planner numbers exactly the tiles of the oracle's
tiling (split blocks first, tiles row-major from each block's top-left)."""
import ctypes
import os
import re

import pytest

import oracle
from tiled_newton_schulz_b200 import himuon

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from tiled_newton_schulz_b200 import build
    build.build()
    return himuon.load()


def header_functions():
    src = open(os.path.join(ROOT, "include", "himuon.h")).read()
    return sorted(set(re.findall(r"HIMUON_API\s+[\w\s\*]+?\b(himuon_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 9
    for name in names:
        assert hasattr(lib, name), name
    assert set(himuon.EXPORTS) <= set(names)


def test_version_and_status_strings(lib):
    assert lib.himuon_version() == 2
    assert himuon.status_string(0) == "ok"
    assert "workspace" in himuon.status_string(-3)


@pytest.mark.parametrize("shapes,splits,T", [
    ([(10, 7)], None, 4),
    ([(8, 24), (5, 5)], [(1, (8, 8, 8)), None], 4),
    ([(300, 500), (128, 128)], None, 128),
    ([(4096, 12288)], [(1, (4096, 4096, 4096))], 128),
    ([(11008, 4096), (4096, 11008)], None, 512),
    ([(10, 6)], [(0, (3, 7))], 4),
    ([(9, 13)], None, 0),
])
def test_planner_matches_oracle_tiling(lib, shapes, splits, T):
    got = himuon.plan_tiles(shapes, splits, T)
    want = []
    for i, shp in enumerate(shapes):
        sp = splits[i] if splits else None
        for (r0, c0, h, w) in oracle.split_blocks(shp, sp):
            TT = max(h, w) if T <= 0 else T
            for (tr, tc, th, tw) in oracle.tile_grid(h, w, TT):
                want.append((i, r0 + tr, c0 + tc, th, tw))
    assert got == want


def test_llama7b_tile_count(lib):
    from tiled_newton_schulz_b200 import inputs
    wl = inputs.llama7b_set(1)
    shapes = [(m.rows, m.cols) for m in wl.matrices]
    splits = [m.split for m in wl.matrices]
    assert len(himuon.plan_tiles(shapes, splits, 128)) == 395264 // 32
    assert len(himuon.plan_tiles(shapes, splits, 256)) == 98816 // 32


def test_invalid_arguments_are_rejected_on_the_host(lib):
    p = himuon.params(128, (3.4445, -4.7750, 2.0315), steps=5)
    m = (himuon.Mat * 1)(himuon.Mat(0, 16, 16, 16, himuon.BF16))   # null data
    rc = lib.himuon_ns_tiled(m, m, 1, None, ctypes.byref(p), None, 0, None)
    assert rc == -1
    good = (himuon.Mat * 1)(himuon.Mat(0x1000, 16, 16, 8, himuon.BF16))   # ld < cols
    assert lib.himuon_ns_tiled(good, good, 1, None, ctypes.byref(p), None, 0, None) == -1
    bad_k = himuon.params(128, [(1.0, 0.0, 0.0)] * 17)
    ok = (himuon.Mat * 1)(himuon.Mat(0x1000, 16, 16, 16, himuon.BF16))
    assert lib.himuon_ns_tiled(ok, ok, 1, None, ctypes.byref(bad_k), None, 0, None) == -2
    split = himuon._splits([(1, (8, 4))], 1)[0]    # sizes do not sum to 16
    assert lib.himuon_workspace_size(ok, 1, split, ctypes.byref(p), 0) == -1


def test_workspace_size_on_the_host(lib):
    import torch
    p = himuon.params(128, (3.4445, -4.7750, 2.0315), steps=5)
    shapes = [(4096, 4096)]
    mats = (himuon.Mat * 1)(himuon.Mat(0x1000, 4096, 4096, 4096, himuon.BF16))
    assert lib.himuon_workspace_size(mats, 1, None, ctypes.byref(p), 0) == 0       # on-chip path
    p256 = himuon.params(256, (3.4445, -4.7750, 2.0315), steps=5)
    assert lib.himuon_workspace_size(mats, 1, None, ctypes.byref(p256), 0) == 0    # on chip, CTA pairs
    p256f = himuon.params(256, (3.4445, -4.7750, 2.0315), steps=5, compute=himuon.FP32)
    assert lib.himuon_workspace_size(mats, 1, None, ctypes.byref(p256f), 0) > 0    # fp32: staged
    p512 = himuon.params(512, (3.4445, -4.7750, 2.0315), steps=5)
    need = lib.himuon_workspace_size(mats, 1, None, ctypes.byref(p512), 0)
    assert need > 512 * 512 * 4 * 64                        # at least the two 16-bit iterates of the 64 tiles
    pc = himuon.params(512, (3.4445, -4.7750, 2.0315), steps=5, chunk_bytes=64 << 20)
    assert lib.himuon_workspace_size(mats, 1, None, ctypes.byref(pc), 0) <= 64 << 20


@pytest.mark.parametrize("op,compute,expect_mib", [
    # 16-bit operand ping-pong 2 x 8 MiB, A and Bop 2 x 2 MiB: no fp32 X (bf16 NS
    # scales in its first products, fp16 NS writes the scaled operand in a second
    # pass over the input, and both last products write the caller's buffer)
    (himuon.OP_NS_FULL, himuon.BF16, 20),
    (himuon.OP_NS_FULL, himuon.FP16, 20),
    (himuon.OP_MOMENTUM_STEP, himuon.BF16, 20),
    # the fp16 momentum step normalises from an fp32 X (16 MiB)
    (himuon.OP_MOMENTUM_STEP, himuon.FP16, 36),
    # Gram NS in fp16: operands 16, R fp32 + fp16 6, RZ fp32 4, Q x 2, Z, RZ fp16 8
    (himuon.OP_GRAM_NS, himuon.FP16, 34),
    # fp32: X x 2 32, A and B 8; Gram adds RZ, Q, Z, a second Q (fp32)
    (himuon.OP_NS_FULL, himuon.FP32, 40),
    (himuon.OP_GRAM_NS, himuon.FP32, 52),
])
def test_staged_workspace_layout_on_the_host(lib, op, compute, expect_mib):
    """The staged workspace of one 1024 x 4096 matrix, whole (n = 1024, m =
    4096, one tile), buffer by buffer: a path that reads the fp32 X must have
    one of its own (its offset would otherwise alias the 16-bit operand), and
    the paths that never touch it must not pay for it.  768 B of per-tile
    partial sums and scales come on top."""
    mats = (himuon.Mat * 1)(himuon.Mat(0x1000, 1024, 4096, 4096, himuon.BF16))
    p = himuon.params(0, (3.4445, -4.7750, 2.0315), steps=5, compute=compute, restart=(3,) if op == himuon.OP_GRAM_NS else ())
    assert lib.himuon_workspace_size(mats, 1, None, ctypes.byref(p), op) == expect_mib * (1 << 20) + 768


def test_per_matrix_tiles_on_the_host(lib):
    """p->tiles: the workspace is the largest group's need; the fixed-scratch
    entry point rejects it; a bad matrix in any group fails the whole call."""
    Q = (3.4445, -4.7750, 2.0315)
    shapes = [(4096, 4096), (1024, 4096), (2048, 2048)]
    mats = (himuon.Mat * 3)(*[himuon.Mat(0x1000 * (i + 1), r, c, c, himuon.BF16) for i, (r, c) in enumerate(shapes)])
    one = lambda i: (himuon.Mat * 1)(mats[i])
    per = []
    for i, T in enumerate((128, 512, 0)):
        per.append(lib.himuon_workspace_size(one(i), 1, None, ctypes.byref(himuon.params(T, Q, steps=5)),
                                             himuon.OP_NS_TILED if T > 0 else himuon.OP_NS_FULL))
    assert per[0] == 0 and per[1] > 0 and per[2] > 0
    pt = himuon.params(128, Q, steps=5, tiles=[128, 512, 0])
    for op in (himuon.OP_NS_TILED, himuon.OP_MOMENTUM_STEP):
        assert lib.himuon_workspace_size(mats, 3, None, ctypes.byref(pt), op) == max(per)
    # all on chip -> no workspace; ns_full ignores tiles
    assert lib.himuon_workspace_size(mats, 3, None, ctypes.byref(himuon.params(0, Q, steps=5, tiles=[128] * 3)),
                                     himuon.OP_NS_TILED) == 0
    assert lib.himuon_workspace_size(mats, 3, None, ctypes.byref(himuon.params(0, Q, steps=5, tiles=[128, 256, 64])),
                                     himuon.OP_NS_TILED) == 0
    full = lib.himuon_workspace_size(mats, 3, None, ctypes.byref(himuon.params(0, Q, steps=5)), himuon.OP_NS_FULL)
    assert lib.himuon_workspace_size(mats, 3, None, ctypes.byref(pt), himuon.OP_NS_FULL) == full
    assert lib.himuon_ns_static(mats, mats, 3, None, ctypes.byref(pt), None) == -2
    bad = (himuon.Mat * 3)(mats[0], mats[1], himuon.Mat(0, 2048, 2048, 2048, himuon.BF16))
    assert lib.himuon_ns_tiled(bad, bad, 3, None, ctypes.byref(pt), None, 0, None) == -1


def test_binding_checks_the_tile_list_length(lib):
    """The C side reads one T per matrix from params.tiles; the binding
    refuses a list of another length before calling it."""
    import torch
    Q = (3.4445, -4.7750, 2.0315)
    x = [torch.zeros(16, 16, dtype=torch.bfloat16) for _ in range(3)]
    with pytest.raises(ValueError):
        himuon.workspace_size(x, himuon.params(128, Q, steps=5, tiles=[128, 256]), himuon.OP_NS_TILED)
    with pytest.raises(ValueError):
        himuon.ns_tiled(x, x, himuon.params(128, Q, steps=5, tiles=[128] * 4))
    assert himuon.workspace_size(x, himuon.params(128, Q, steps=5, tiles=[128, 0, 256]), himuon.OP_NS_TILED) >= 0
