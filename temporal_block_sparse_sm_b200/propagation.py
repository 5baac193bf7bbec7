"""How the skip mask is carried across denoising steps.

"LiteAttention: Temporal Sparse Attention for Diffusion Transformers" (skill
page), Core Concept: the mask is computed early with QK-Skip, carried forward
across timesteps, and updated only if the attention pattern diverges
significantly; Architecture Overview, Persistent Propagation: decisions carry
forward unless the attention distribution shifts.  Every policy below drives
the same step kernel through the C ABI; they differ only in which mask each
step reads and writes:

``propagate``
    QK-Skip at every step on the live tiles; dead tiles stay dead (the mask is
    AND-accumulated in place).
``recompute``
    the mask is reset to all-live before every step (QK-Skip decides afresh).
``early``
    QK-Skip only during the first ``early_steps`` steps, then the mask is
    frozen: from then on the threshold is -inf, so the test can kill nothing and
    each step computes exactly the frozen live tiles.  This is a schedule, see
    :func:`early_only_schedule`.
``refresh``
    propagate, and every ``every`` steps a probe step runs from an all-live
    mask into a second mask.  The divergence is the share of the probe's live
    tiles that the propagated mask has lost (tiles propagation can never
    revive).  Above ``revive`` the probe's mask replaces the propagated one;
    otherwise propagation continues from the mask it had.  The probe step's
    output is the output of that step either way.

The pages give no divergence measure or threshold; the share of revivable
tiles is the plainest measure the mask store can give exactly
(``lite_attn_mask_compare``).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

POLICIES = ("propagate", "recompute", "early", "refresh")


def early_only_schedule(taus: Sequence[float], early_steps: int) -> list:
    """The schedule of the ``early`` policy: taus[t] for t < early_steps, then -inf."""
    if early_steps < 0:
        raise ValueError("early_steps must be >= 0")
    return [float(t) if i < early_steps else -math.inf for i, t in enumerate(taus)]


class MaskPolicy:
    """Runs the steps of one attention call of a denoising trajectory under a policy.

    ``plan`` is a :class:`~temporal_block_sparse_sm_b200.liteattn.Plan`; for the
    ``early`` policy its schedule must come from :func:`early_only_schedule`.
    """

    def __init__(self, plan, policy: str = "propagate", every: int = 0, revive: float = 0.0):
        if policy not in POLICIES:
            raise ValueError(f"policy must be one of {POLICIES}")
        if policy == "refresh" and every < 1:
            raise ValueError("the refresh policy needs every >= 1")
        if not 0.0 <= revive <= 1.0:
            raise ValueError("revive is a fraction in [0, 1]")
        self.plan, self.policy, self.every, self.revive = plan, policy, every, revive
        self.mask = plan.mask()
        self.probe = plan.mask() if policy == "refresh" else None
        self.history = []

    def is_probe_step(self, t: int) -> bool:
        return self.policy == "refresh" and t > 0 and t % self.every == 0

    def start(self, stream=None):
        """Begin a trajectory: the mask becomes all-live."""
        self.mask.reset(stream)
        self.history = []

    def step(self, q, k, v, o, t: int, stream=None) -> dict:
        """Step t; returns what the policy did ({"t", "probe", "adopted", "divergence"})."""
        info = {"t": t, "probe": False, "adopted": False, "divergence": None}
        if self.policy == "recompute":
            self.mask.reset(stream)
        if self.is_probe_step(t):
            self.probe.reset(stream)
            self.plan.step(q, k, v, o, self.probe, self.probe, t, stream)
            only_probe, _ = self.probe.compare(self.mask, stream)
            live_probe = self.plan.stats(self.probe)["live_out"]
            div = only_probe / live_probe if live_probe else 0.0
            info.update(probe=True, divergence=div)
            if div > self.revive:
                self.mask, self.probe = self.probe, self.mask
                info["adopted"] = True
        else:
            self.plan.step(q, k, v, o, self.mask, self.mask, t, stream)
        self.history.append(info)
        return info

    def close(self):
        for m in (self.mask, self.probe):
            if m is not None:
                m.close()
