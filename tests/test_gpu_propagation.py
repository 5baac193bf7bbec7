"""GPU: mask comparison (lite_attn_mask_compare) and the propagation policies.

The comparison is integer work, checked bit-exactly against numpy popcounts.
The policies run the step kernel on seeded workloads; every step is checked
against the oracle on the mask that step actually read, and each refresh
decision against the divergence recomputed from the exported masks.
"""
from __future__ import annotations


import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn, synthetic
from temporal_block_sparse_sm_b200.propagation import MaskPolicy, early_only_schedule
from tests.parity import check_step, pick_items

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def _popcount(bits: np.ndarray) -> int:
    return int(np.unpackbits(np.ascontiguousarray(bits, dtype=np.uint32).view(np.uint8)).sum())


@pytest.mark.parametrize("B,H,N,bc", [(1, 12, 8192, 128), (2, 3, 1000, 64), (1, 2, 70000, 64), (1, 1, 1, 64)])
def test_compare_matches_numpy(B, H, N, bc):
    plan = liteattn.Plan(B, H, N, bc, bc, bc, [-1.0])
    a, b = plan.mask(), plan.mask()
    for seed, (fa, fb) in enumerate([(0.5, 0.5), (0.9, 0.1), (1.0, 0.3), (0.0, 0.7)]):
        ba = synthetic.random_live_bits(plan.R, plan.Tk, fa, seed=2 * seed, keep_first=False).numpy().astype(np.uint32)
        bb = synthetic.random_live_bits(plan.R, plan.Tk, fb, seed=2 * seed + 1, keep_first=False).numpy().astype(np.uint32)
        a.import_bits(ba)
        b.import_bits(bb)
        want = (_popcount(ba & ~bb), _popcount(bb & ~ba))
        assert a.compare(b) == want
        assert b.compare(a) == want[::-1]
        assert a.compare(a) == (0, 0)


def test_compare_rejects_masks_of_other_plans():
    p1 = liteattn.Plan(1, 1, 256, 64, 64, 64, [-1.0])
    p2 = liteattn.Plan(1, 1, 256, 64, 64, 64, [-1.0])
    with pytest.raises(liteattn.LiteAttnError) as e:
        p1.mask().compare(p2.mask())
    assert e.value.code == liteattn.LITE_ERR_PLAN_MISMATCH


def _run_policy(cfg, taus, policy, n_items=48, **kw):
    """Run the trajectory under `policy`, checking every step against the oracle."""
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, taus)
    pol = MaskPolicy(plan, policy, **kw)
    wl = synthetic.Workload(cfg, seed=0, device="cuda")
    o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    all_live = plan.mask().export_bits()
    pol.start()
    out = []
    for t in range(len(taus)):
        q, k, v = wl.inputs(t)
        probe = pol.is_probe_step(t)
        bits_in = all_live if (probe or policy == "recompute") else pol.mask.export_bits()
        before = pol.mask.export_bits()
        info = pol.step(q, k, v, o, t)
        written = pol.mask if (info["adopted"] or not probe) else pol.probe
        bits_out = written.export_bits()
        items = np.arange(plan.R) if n_items is None else pick_items(cfg.B, cfg.H, plan.Tq, n_items, 77 + t)
        res = check_step(q, k, v, o, bits_in, bits_out, B=cfg.B, H=cfg.H, N=cfg.N, d=cfg.d, Br=cfg.Br, Bc=cfg.Bc,
                         tau=plan.taus[t], items=items, step=t)
        if probe:
            only = _popcount(bits_out & ~before)
            assert info["divergence"] == pytest.approx(only / max(1, _popcount(bits_out)), abs=1e-12)
            assert info["adopted"] == (info["divergence"] > kw.get("revive", 0.0))
        out.append((info, res, _popcount(pol.mask.export_bits())))
    return plan, pol, out


def test_early_policy_freezes_the_mask_c2():
    cfg = synthetic.CONFIGS["c2"]
    taus = early_only_schedule(cfg.taus(), 2)
    plan, pol, out = _run_policy(cfg, taus, "early")
    live = [n for _, _, n in out]
    print("live tiles by step", live, "of", plan.R * plan.Tk)
    assert all(n == live[1] for n in live[2:]), "the mask changed after the early steps"
    st = plan.stats(pol.mask)
    assert st["newly_dead"] == 0 and st["live_in"] == st["live_out"]


@pytest.mark.parametrize("revive", [0.0, 1.0])
def test_refresh_policy_c2(revive):
    cfg = synthetic.CONFIGS["c2"]
    plan, pol, out = _run_policy(cfg, cfg.taus(), "refresh", every=3, revive=revive)
    probes = [info for info, _, _ in out if info["probe"]]
    assert [p["t"] for p in probes] == [3, 6, 9]
    if revive == 1.0:
        assert not any(p["adopted"] for p in probes)
    print([(p["t"], round(p["divergence"], 4), p["adopted"]) for p in probes])


def test_recompute_policy_c1_every_item():
    cfg = synthetic.CONFIGS["c1"]
    _run_policy(cfg, cfg.taus(), "recompute", n_items=None)
