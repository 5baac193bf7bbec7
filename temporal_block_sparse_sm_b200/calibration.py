"""Accumulated-error calibration of the per-step QK-Skip threshold.

"LiteAttention: Temporal Sparse Attention for Diffusion Transformers" (skill
page), Architecture Overview: the method assigns variable error budgets to
timesteps, early steps tolerating less error.  The pages give no formula, so
this module takes the plainest reading that the rest supports:

* a **budget** bounds, per step t, the relative L1 error of that step's
  attention output against dense attention on the same inputs,
  sum |o_t - dense_t| / sum |dense_t| <= eps_t, with eps_t growing with t
  (:func:`error_budgets`);
* **calibration** walks the steps of a calibration trajectory in order and,
  at each step, picks the most aggressive threshold of a grid whose output,
  computed from the mask carried over from the calibrated earlier steps, stays
  within that step's budget.  The error measured therefore includes what the
  earlier steps' decisions still cost (tiles dead on entry), hence
  "accumulated".  When no grid value fits, the step runs with tau = -inf
  (nothing more dies) and its error is recorded as over budget.

The result is a threshold schedule for :class:`liteattn.Plan`.  Every step,
error and mask operation runs in the CUDA library (``lite_attn_step``,
``lite_attn_output_error``, the mask store); this module only chooses.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, List, Sequence


def error_budgets(T: int, total: float, growth: str = "linear") -> List[float]:
    """Per-step budgets summing to `total`, non-decreasing in t (early steps tighter).

    growth = "linear": eps_t proportional to t + 1; "flat": equal budgets."""
    if T < 1 or not total > 0:
        raise ValueError("need T >= 1 and a positive total budget")
    if growth == "linear":
        w = [t + 1.0 for t in range(T)]
    elif growth == "flat":
        w = [1.0] * T
    else:
        raise ValueError("growth must be 'linear' or 'flat'")
    s = sum(w)
    return [total * x / s for x in w]


def threshold_grid(lo: float = 1e-8, hi: float = 1e-1, per_decade: int = 1) -> List[float]:
    """Candidate thresholds ln(1e-8) ... ln(1e-1), most aggressive first, then -inf."""
    n = int(round(math.log10(hi / lo) * per_decade))
    g = [math.log(hi) - i * (math.log(hi) - math.log(lo)) / n for i in range(n + 1)]
    return g + [-math.inf]


@dataclass
class Calibration:
    taus: List[float] = field(default_factory=list)       # chosen threshold per step
    errors: List[float] = field(default_factory=list)     # relative L1 error of each step's output
    budgets: List[float] = field(default_factory=list)
    over_budget: List[int] = field(default_factory=list)  # steps where even tau = -inf exceeded the budget
    trials: int = 0                                       # steps run while searching


def calibrate(grid_plan, dense_plan, inputs: Callable[[int], tuple], budgets: Sequence[float],
              new_output: Callable[[], object]) -> Calibration:
    """Choose tau_t for each step of the trajectory `inputs(t)`, t < len(budgets).

    grid_plan  : a Plan whose threshold schedule is the candidate grid, most aggressive
                 first and ending with -inf (step index = grid index);
    dense_plan : a Plan of the same shape with schedule [-inf] (the dense reference);
    new_output : allocates an output tensor of the plans' shape.
    """
    grid = grid_plan.taus
    if not grid or not (math.isinf(grid[-1]) and grid[-1] < 0):
        raise ValueError("the grid must end with -inf")
    if any(b >= a for a, b in zip(grid, grid[1:])):
        raise ValueError("the grid must be strictly decreasing (most aggressive first)")
    cur, trial = grid_plan.mask(), grid_plan.mask()
    dmask = dense_plan.mask()
    o_dense, o_try = new_output(), new_output()
    res = Calibration(budgets=list(budgets))
    cur.reset()
    for t, eps in enumerate(budgets):
        q, k, v = inputs(t)
        dmask.reset()
        dense_plan.step(q, k, v, o_dense, dmask, dmask, 0)
        carried = cur.export_bits()
        chosen, err = None, None
        for gi in range(len(grid)):
            trial.import_bits(carried)
            grid_plan.step(q, k, v, o_try, trial, trial, gi)
            res.trials += 1
            err = grid_plan.output_error(o_try, o_dense)["rel_l1"]
            if err <= eps or gi == len(grid) - 1:
                chosen = gi
                break
        if err > eps:
            res.over_budget.append(t)
        res.taus.append(grid[chosen])
        res.errors.append(err)
        cur, trial = trial, cur
    return res
