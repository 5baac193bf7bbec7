"""Host logic of the threshold calibration, on a fake plan (no GPU).

The fake step kills a fixed number of tiles per grid index and reports an
error of 1e-4 per dead tile, so every choice of the calibration can be
worked out by hand.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

from temporal_block_sparse_sm_b200.calibration import calibrate, error_budgets, threshold_grid

GRID = [math.log(0.1), math.log(0.01), math.log(0.001), -math.inf]
KILLS = [5, 2, 1, 0]          # tiles killed by grid index 0..3


class FakeMask:
    def __init__(self):
        self.dead = 0

    def reset(self):
        self.dead = 0

    def export_bits(self):
        return np.array([self.dead])

    def import_bits(self, bits):
        self.dead = int(bits[0])


class FakePlan:
    def __init__(self, taus):
        self.taus = list(taus)
        self.steps = []

    def mask(self):
        return FakeMask()

    def step(self, q, k, v, o, mask_in, mask_out, idx):
        self.steps.append(idx)
        if math.isinf(self.taus[idx]) and len(self.taus) == 1:     # the dense plan
            o["err"] = 0.0
            return
        mask_out.dead = mask_in.dead + KILLS[idx]
        o["err"] = 1e-4 * mask_out.dead

    def output_error(self, o, o_ref):
        return {"rel_l1": o["err"]}


def _calibrate(budgets):
    gp, dp = FakePlan(GRID), FakePlan([-math.inf])
    return calibrate(gp, dp, lambda t: (None, None, None), budgets, dict), gp, dp


def test_picks_the_most_aggressive_threshold_within_each_budget():
    res, gp, dp = _calibrate([3.5e-4, 4e-4, 1e-4])
    # step 0: 5 dead -> 5e-4 too much; 2 dead -> 2e-4 fits.  step 1: 2 + 5 too much; 2 + 2 = 4e-4 fits
    # (budget inclusive).  step 2: 4 carried already cost 4e-4 > 1e-4: -inf, over budget.
    assert res.taus == [GRID[1], GRID[1], -math.inf]
    assert res.errors == pytest.approx([2e-4, 4e-4, 4e-4])
    assert res.over_budget == [2]
    assert res.trials == 2 + 2 + 4
    assert dp.steps == [0, 0, 0]                      # one dense reference step per step


def test_generous_budgets_take_the_most_aggressive_value():
    res, *_ = _calibrate([1.0, 1.0])
    assert res.taus == [GRID[0], GRID[0]] and res.trials == 2 and not res.over_budget


def test_error_budgets_grow_and_sum_to_total():
    b = error_budgets(10, 2e-3)
    assert sum(b) == pytest.approx(2e-3)
    assert all(x < y for x, y in zip(b, b[1:]))
    assert b[-1] == pytest.approx(10 * b[0])
    assert error_budgets(4, 1.0, "flat") == [0.25] * 4
    with pytest.raises(ValueError):
        error_budgets(0, 1.0)
    with pytest.raises(ValueError):
        error_budgets(3, 1.0, "cubic")


def test_threshold_grid_order_and_end():
    g = threshold_grid()
    assert g[0] == pytest.approx(math.log(0.1)) and g[-2] == pytest.approx(math.log(1e-8))
    assert math.isinf(g[-1]) and g[-1] < 0
    assert all(b < a for a, b in zip(g, g[1:]))


def test_grid_must_end_with_minus_infinity_and_decrease():
    with pytest.raises(ValueError):
        calibrate(FakePlan(GRID[:-1]), FakePlan([-math.inf]), lambda t: (None,) * 3, [1.0], dict)
    with pytest.raises(ValueError):
        calibrate(FakePlan([GRID[1], GRID[0], -math.inf]), FakePlan([-math.inf]), lambda t: (None,) * 3, [1.0], dict)
