"""Runtime tile-size schedules (host logic, no GPU): the step/matrix schedule
and the budgeted choice of tile sizes from a cost table."""
import itertools
import math

import pytest

from tiled_newton_schulz_b200.schedule import (TileSchedule, choose_tiles, modeled_cost, pareto_chain, quality)


def test_quality_orders_whole_matrix_last():
    assert sorted([512, 0, 32, 128, -1], key=quality) == [32, 128, 512, 0, -1]


def test_schedule_milestones_and_overrides():
    s = TileSchedule(default=128, milestones=[(1000, 256), (10, 64)], per_matrix={2: 0, 3: [(500, 32)]})
    assert s.tiles(0, 4) == [128, 128, 0, 128]
    assert s.tiles(10, 4) == [64, 64, 0, 64]
    assert s.tiles(999, 4) == [64, 64, 0, 32]
    assert s.tiles(1000, 5) == [256, 256, 0, 32, 256]
    import numpy as np
    assert TileSchedule(per_matrix={0: np.int64(256)}).tiles(0, 2) == [256, 128]
    with pytest.raises(ValueError):
        TileSchedule(milestones=[(5, 64), (5, 128)])
    with pytest.raises(ValueError):
        TileSchedule(milestones=[(-1, 64)])


def test_pareto_chain_drops_dominated_candidates():
    # T = 32 costs more than T = 128 (redundant work on chip): never worth it
    ch = pareto_chain({32: 4.0, 64: 2.0, 128: 1.0, 256: 8.0, 512: 9.0, 0: 9.0})
    assert ch == [(128, 1.0), (256, 8.0), (0, 9.0)]
    with pytest.raises(ValueError):
        pareto_chain({128: float("nan")})


COSTS = [
    {32: 4.0, 64: 2.0, 128: 1.0, 256: 8.0, 512: 9.0, 0: 12.0},
    {64: 0.5, 128: 0.3, 256: 2.0, 0: 6.0},
    {128: 1.0, 256: 1.5, 512: 2.5},
]
BUDGETS = [0.0, 2.3, 2.8, 3.0, 4.0, 5.0, 9.9, 12.0, 15.0, 20.0, 100.0]


@pytest.mark.parametrize("budget", BUDGETS)
def test_choose_tiles_fits_budget_and_stops_only_when_no_upgrade_fits(budget):
    got = choose_tiles(COSTS, budget)
    chains = [pareto_chain(c) for c in COSTS]
    cheapest = sum(ch[0][1] for ch in chains)
    if budget < cheapest:
        assert got == [ch[0][0] for ch in chains]
        return
    total = modeled_cost(COSTS, got)
    assert total <= budget
    for T, ch in zip(got, chains):
        ts = [t for t, _ in ch]
        assert T in ts                                   # on the Pareto chain
        k = ts.index(T)
        if k + 1 < len(ch):                              # the next upgrade does not fit
            assert total + ch[k + 1][1] - ch[k][1] > budget


def test_choose_tiles_is_monotone_in_budget():
    prev = None
    for budget in BUDGETS:
        got = choose_tiles(COSTS, budget)
        if prev is not None:
            assert all(quality(a) >= quality(b) for a, b in zip(got, prev))
        prev = got


def test_choose_tiles_brute_force_small():
    """On a tiny set, the greedy result is never beaten on every matrix at
    once by another choice that also fits (exhaustive search)."""
    for budget in BUDGETS:
        got = choose_tiles(COSTS, budget)
        if modeled_cost(COSTS, got) > budget:
            continue
        for ch in itertools.product(*[list(c) for c in COSTS]):
            if modeled_cost(COSTS, ch) > budget:
                continue
            better_everywhere = all(quality(a) > quality(b) for a, b in zip(ch, got))
            assert not better_everywhere, (budget, got, ch)


def test_choose_tiles_extremes():
    assert choose_tiles(COSTS, math.inf) == [0, 0, 512]
    assert choose_tiles(COSTS, 0.0) == [128, 128, 128]
    assert choose_tiles([], 1.0) == []
    with pytest.raises(ValueError):
        choose_tiles([{}], 1.0)


def test_choose_tiles_takes_cheapest_upgrade_first():
    # budget for exactly one upgrade: matrix 2 (128 -> 256, +0.5) before matrix 1 (128 -> 256, +1.7)
    assert choose_tiles(COSTS, 2.3 + 0.5) == [128, 128, 256]
    assert choose_tiles(COSTS, 2.3 + 0.5 + 1.0) == [128, 128, 512]
