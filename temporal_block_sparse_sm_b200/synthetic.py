"""Seeded synthetic video-token workloads for LiteAttention.

This module holds only input generation: positions on a (frame, y, x) grid, a
sinusoidal 3D positional feature, seeded Gaussian noise, per-step perturbation
and drift, and the threshold schedules of each workload.  It holds none of the
attention method's arithmetic, so both the CUDA path and the CPU oracle can
consume its tensors.

Recipe (the pages name production video diffusion transformers -- "LiteAttention:
A Temporal Sparse Attention for Diffusion Transformers", abstract -- but ship no
data; these seeded tensors stand in for their attention inputs):

* token n sits at (f, y, x) with n = (f*Y + y)*X + x;
* phi(pos) in R^d has d/2 cos/sin pairs; pair p uses axis a = p mod 3 and rank
  k = p // 3 among that axis's K_a pairs, with angular rate
  w = L_a ** (-k / K_a) rad/token (L_a = extent of axis a);
  phi[2p] = cos(w*pos_a), phi[2p+1] = sin(w*pos_a);
* base tensors q0 = 2*phi + 0.5*N(0,1), k0 = 2*phi + 0.5*N(0,1) (independent
  noise for every batch and head), v0 ~ N(0,1);
* step t: x_t = x0 + sigma*eps_t + c*t*drift_x, eps_t fresh per step,
  drift_x ~ N(0,1) fixed per seed; rounded to bf16 after the sum.

Every random tensor comes from its own ``torch.Generator`` seeded from
(seed, tensor id, step), so any step can be produced without the ones before.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    B: int
    H: int
    N: int
    d: int
    Br: int
    Bc: int
    grid: Tuple[int, int, int]
    T: int
    sigma: float
    drift: float
    schedule: Tuple[str, float, float] = ("const", math.log(1e-4), math.log(1e-4))
    fixed_taus: Tuple[float, ...] = field(default_factory=tuple)

    def taus(self) -> List[float]:
        """Per-step thresholds (natural log), length T."""
        kind, a, b = self.schedule
        if kind == "const":
            return [float(a)] * self.T
        if kind == "loglinear":
            if self.T == 1:
                return [float(a)]
            return [float(a + (b - a) * t / (self.T - 1)) for t in range(self.T)]
        raise ValueError(kind)


LN = math.log
CONFIGS = {
    # small case: 4x16x16 grid, d=64, 64-wide tiles, 3 steps at ln(1e-4)
    "c1": WorkloadConfig("c1-N1024-H2-d64", 1, 2, 1024, 64, 64, 64, (4, 16, 16), 3, 0.05, 0.0,
                         ("const", LN(1e-4), LN(1e-4))),
    # 8x32x32 grid, 12 heads, d=128, 10 steps, ln(1e-6) -> ln(1e-3)
    "c2": WorkloadConfig("c2-N8192-H12-d128", 1, 12, 8192, 128, 128, 128, (8, 32, 32), 10, 0.03, 0.0,
                         ("loglinear", LN(1e-6), LN(1e-3))),
    # 1.3B video-DiT attention shape: 21x30x52 grid
    "c3": WorkloadConfig("c3-N32760-H12-d128", 1, 12, 32760, 128, 128, 128, (21, 30, 52), 50, 0.02, 0.01,
                         ("loglinear", LN(1e-6), LN(1e-3))),
    # 720p video-DiT attention shape: 30x45x80 grid, 24 heads
    "c4": WorkloadConfig("c4-N108000-H24-d128", 1, 24, 108000, 128, 128, 128, (30, 45, 80), 50, 0.02, 0.01,
                         ("loglinear", LN(1e-6), LN(1e-3))),
    # skip-rate sweep on the 1.3B shape, 20 steps, fixed thresholds
    "c5": WorkloadConfig("c5-N32760-H12-d128-sweep", 1, 12, 32760, 128, 128, 128, (21, 30, 52), 20, 0.02,
                         0.01, ("const", LN(1e-4), LN(1e-4)),
                         (LN(1e-8), LN(1e-5), LN(1e-4), LN(1e-3), LN(1e-2), -math.inf)),
}


def positions(grid: Tuple[int, int, int]) -> torch.Tensor:
    """(N, 3) integer (f, y, x) positions in row-major token order."""
    F, Y, X = grid
    f = torch.arange(F).repeat_interleave(Y * X)
    y = torch.arange(Y).repeat_interleave(X).repeat(F)
    x = torch.arange(X).repeat(F * Y)
    return torch.stack([f, y, x], dim=1)


def phi(grid: Tuple[int, int, int], d: int) -> torch.Tensor:
    """Sinusoidal 3D positional feature, (N, d) float64, |phi|^2 = d/2."""
    if d % 2:
        raise ValueError("d must be even")
    pos = positions(grid).to(torch.float64)
    pairs = d // 2
    counts = [len(range(a, pairs, 3)) for a in range(3)]
    out = torch.empty(pos.shape[0], d, dtype=torch.float64)
    for p in range(pairs):
        a = p % 3
        rank = p // 3
        L = float(grid[a])
        w = L ** (-rank / counts[a]) if L > 1 else 1.0
        out[:, 2 * p] = torch.cos(w * pos[:, a])
        out[:, 2 * p + 1] = torch.sin(w * pos[:, a])
    return out


def _gen(device, seed: int, tensor_id: int, step: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tensor_id * 7_919 + step * 104_729) & 0x7FFF_FFFF_FFFF)
    return g


class Workload:
    """Seeded inputs of one configuration on one device.

    ``inputs(t)`` returns bf16 (q, k, v) of shape [B, H, N, d] for step t.
    """

    Q, K, V = 0, 1, 2

    def __init__(self, cfg: WorkloadConfig, seed: int = 0, device="cpu"):
        self.cfg = cfg
        self.seed = seed
        self.device = torch.device(device)
        shape = (cfg.B, cfg.H, cfg.N, cfg.d)
        ph = (2.0 * phi(cfg.grid, cfg.d)).to(torch.float32).to(self.device)
        self.base = []
        for tid in (self.Q, self.K, self.V):
            noise = torch.randn(shape, generator=_gen(self.device, seed, tid), device=self.device,
                                dtype=torch.float32)
            if tid == self.V:
                self.base.append(noise)
            else:
                self.base.append(ph + 0.5 * noise)
        self.drift = None
        if cfg.drift:
            self.drift = [torch.randn(shape, generator=_gen(self.device, seed, 10 + tid), device=self.device,
                                      dtype=torch.float32) for tid in (self.Q, self.K, self.V)]

    @property
    def shape(self):
        c = self.cfg
        return (c.B, c.H, c.N, c.d)

    def inputs(self, t: int, out: Optional[Tuple[torch.Tensor, ...]] = None):
        c = self.cfg
        res = []
        for tid in (self.Q, self.K, self.V):
            x = self.base[tid].clone()
            eps = torch.randn(self.shape, generator=_gen(self.device, self.seed, 100 + tid, t + 1),
                              device=self.device, dtype=torch.float32)
            x.add_(eps, alpha=c.sigma)
            if self.drift is not None:
                x.add_(self.drift[tid], alpha=c.drift * t)
            xb = x.to(torch.bfloat16)
            if out is not None:
                out[tid].copy_(xb)
                res.append(out[tid])
            else:
                res.append(xb)
        return tuple(res)


def random_live_bits(rows: int, Tk: int, live_fraction: float, seed: int, keep_first: bool = True,
                     device="cpu") -> torch.Tensor:
    """Random imported masks: each tile live with probability ``live_fraction``.

    Returns int64 tensor [rows, W] holding the uint32 words (bits >= Tk are 0).
    """
    g = _gen(device, seed, 999)
    live = torch.rand(rows, Tk, generator=g, device=device) < live_fraction
    if keep_first:
        live[:, 0] = True
    W = -(-Tk // 32)
    pad = torch.zeros(rows, W * 32, dtype=torch.int64, device=device)
    pad[:, :Tk] = live.to(torch.int64)
    weights = (torch.ones(32, dtype=torch.int64, device=device) << torch.arange(32, device=device))
    return (pad.view(rows, W, 32) * weights).sum(-1)


def locality_live_bits(grid: Tuple[int, int, int], B: int, H: int, Br: int, Bc: int, live_fraction: float) -> torch.Tensor:
    """Locality-structured imported masks: each query tile keeps the key tiles
    nearest to it on the (frame, y, x) token grid.

    A tile's position is the mean position of its tokens; query tile i keeps the
    ceil(live_fraction * Tk) key tiles whose positions are closest (Euclidean, in
    grid units; ties by tile index), which always includes its own diagonal tile
    for live_fraction > 0.  Every (batch, head) gets the same pattern.  This is the
    spatio-temporal sparsity the locality generator produces, at a chosen skip rate.
    Returns int64 tensor [B*H*Tq, W] holding the uint32 words (bits >= Tk are 0).
    """
    pos = positions(grid).to(torch.float64)
    N = pos.shape[0]
    Tq, Tk = -(-N // Br), -(-N // Bc)
    qc = torch.stack([pos[i * Br:min(N, (i + 1) * Br)].mean(0) for i in range(Tq)])
    kc = torch.stack([pos[j * Bc:min(N, (j + 1) * Bc)].mean(0) for j in range(Tk)])
    keep = max(0, min(Tk, math.ceil(live_fraction * Tk)))
    dist = torch.cdist(qc, kc)                                   # [Tq, Tk]
    order = torch.argsort(dist + 1e-9 * torch.arange(Tk, dtype=torch.float64), dim=1)
    live = torch.zeros(Tq, Tk, dtype=torch.bool)
    if keep:
        live.scatter_(1, order[:, :keep], True)
    W = -(-Tk // 32)
    pad = torch.zeros(Tq, W * 32, dtype=torch.int64)
    pad[:, :Tk] = live.to(torch.int64)
    weights = torch.ones(32, dtype=torch.int64) << torch.arange(32)
    rows = (pad.view(Tq, W, 32) * weights).sum(-1)
    return rows.repeat(B * H, 1)
