"""Host logic of the mask-propagation policies, on fake plans and masks (no GPU).

The fake step kills exactly the tiles a hand-written table names for that
step, so each policy's resulting mask and every refresh decision can be
written down in advance.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

from temporal_block_sparse_sm_b200.propagation import MaskPolicy, early_only_schedule

N_TILES = 10


class FakeMask:
    def __init__(self):
        self.live = np.ones(N_TILES, dtype=bool)

    def reset(self, stream=None):
        self.live[:] = True

    def compare(self, other, stream=None):
        return int((self.live & ~other.live).sum()), int((other.live & ~self.live).sum())

    def close(self):
        pass


class FakePlan:
    """step t keeps the live-in tiles not listed in kills[t] (dead stays dead)."""

    def __init__(self, kills):
        self.kills = kills
        self.calls = []

    def mask(self):
        return FakeMask()

    def step(self, q, k, v, o, mask_in, mask_out, t, stream=None):
        keep = np.ones(N_TILES, dtype=bool)
        keep[list(self.kills.get(t, ()))] = False
        self.calls.append((t, mask_in.live.copy()))
        mask_out.live = mask_in.live & keep

    def stats(self, mask):
        return {"live_out": int(mask.live.sum())}


def _live(mask):
    return set(np.flatnonzero(mask.live).tolist())


def _run(policy, kills, T, **kw):
    plan = FakePlan(kills)
    pol = MaskPolicy(plan, policy, **kw)
    pol.start()
    infos = [pol.step(None, None, None, None, t) for t in range(T)]
    return plan, pol, infos


KILLS = {0: (9,), 1: (8, 7), 2: (6,), 3: (5,), 4: (4,), 5: (3,)}


def test_propagate_accumulates_every_kill():
    _, pol, infos = _run("propagate", KILLS, 6)
    assert _live(pol.mask) == {0, 1, 2}
    assert not any(i["probe"] for i in infos)


def test_recompute_keeps_only_the_last_steps_kills():
    plan, pol, _ = _run("recompute", KILLS, 6)
    assert _live(pol.mask) == set(range(10)) - {3}
    assert all(m.all() for _, m in plan.calls)     # every step read an all-live mask


def test_refresh_adopts_the_probe_when_divergence_exceeds_revive():
    # steps 0..2 kill 9, 8, 7, 6; the probe at step 3 starts all-live and kills only 5,
    # so it holds {0..4, 6..9}: 4 of its 9 live tiles (6, 7, 8, 9) are dead in the
    # propagated mask -> divergence 4/9
    plan, pol, infos = _run("refresh", KILLS, 4, every=3, revive=0.4)
    assert infos[3]["probe"] and infos[3]["adopted"]
    assert infos[3]["divergence"] == pytest.approx(4 / 9)
    assert _live(pol.mask) == set(range(10)) - {5}
    assert plan.calls[3][1].all()                    # the probe read an all-live mask


def test_refresh_keeps_propagating_below_revive():
    plan, pol, infos = _run("refresh", KILLS, 5, every=3, revive=0.5)
    assert infos[3]["probe"] and not infos[3]["adopted"]
    # step 3's kill (5) went to the probe only; step 4 continues from the propagated mask
    assert _live(pol.mask) == {0, 1, 2, 3, 5}
    assert set(np.flatnonzero(plan.calls[4][1]).tolist()) == {0, 1, 2, 3, 4, 5}


def test_refresh_probe_steps_are_multiples_of_every():
    _, _, infos = _run("refresh", {}, 10, every=4, revive=0.0)
    assert [i["t"] for i in infos if i["probe"]] == [4, 8]
    assert not any(i["adopted"] for i in infos)      # nothing died: divergence 0, not above 0


def test_early_only_schedule():
    taus = [math.log(1e-4)] * 5
    s = early_only_schedule(taus, 2)
    assert s[:2] == taus[:2] and all(math.isinf(x) and x < 0 for x in s[2:])
    assert early_only_schedule(taus, 0) == [-math.inf] * 5
    assert early_only_schedule(taus, 9) == taus
    with pytest.raises(ValueError):
        early_only_schedule(taus, -1)


@pytest.mark.parametrize("kw", [dict(policy="sometimes"), dict(policy="refresh", every=0),
                                dict(policy="refresh", every=2, revive=1.5)])
def test_policy_argument_checks(kw):
    with pytest.raises(ValueError):
        MaskPolicy(FakePlan({}), **kw)
