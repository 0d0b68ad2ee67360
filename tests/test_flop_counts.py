"""The nominal FLOP count behind every TFLOP/s and roofline figure, pinned to
what the Gram Newton-Schulz page prints (tests/golden/gram_ns_flop_counts.json):
its per-iteration terms of standard NS, their total, and the savings it
reports for naive Gram NS against standard NS with and without symmetric
GEMMs.  A dropped or doubled term in the count fails here."""
import json
import os

import pytest

import bench
from tiled_newton_schulz_b200 import inputs, shard

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "gram_ns_flop_counts.json")))


@pytest.mark.parametrize("h,w", [(128, 128), (64, 256), (256, 64), (1024, 4096), (4096, 11008), (300, 500)])
def test_standard_ns_count_is_the_sum_of_the_printed_terms(h, w):
    n, m = min(h, w), max(h, w)
    K = 5
    terms = 2 * m * n * n + 2 * n ** 3 + 2 * m * n * n       # X X^T, A^2, B X
    assert bench.flops_per_tile(h, w, K) == K * terms
    assert shard.tile_flops(h, w, K) == K * terms


def test_printed_gram_savings_follow_from_the_count():
    n, alpha, T = 1024, 4, 5
    m = alpha * n
    standard = bench.flops_per_tile(n, m, T)                  # 2(2 alpha + 1) n^3 per iteration
    standard_sym = T * (m * n * n + n ** 3 + 2 * m * n * n)   # X X^T and A^2 as half products
    gram = (4 * T + 3 * alpha - 3) * n ** 3
    got = GOLDEN["printed_savings_of_naive_gram_ns"]
    tol = GOLDEN["printed_precision"] / 2
    assert abs((1 - gram / standard) - got["vs_standard_without_symmetric_gemm"]) <= tol
    assert abs((1 - gram / standard_sym) - got["vs_standard_with_symmetric_gemm"]) <= tol


def test_workload_counts_of_the_7b_set():
    wl = inputs.llama7b_set(32)
    mats = [((m.rows, m.cols), m.split) for m in wl.matrices]
    tiles, flops = bench.workload_tiles(mats, 128)
    assert tiles == 395264
    assert flops == 30 * 128 * wl.elements                    # 6 T^3 per step per square tile, K = 5
    assert abs(flops - 2.49e13) / 2.49e13 < 0.005
    tiles256, flops256 = bench.workload_tiles(mats, 256)
    assert tiles256 == 98816 and flops256 == 2 * flops
