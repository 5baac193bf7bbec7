"""Property-based pins of the CPU oracle (CPU, hypothesis).

The fixed-case pins in test_oracle_pins.py are repeated here over randomly
drawn small problems: any N (ragged last tiles), odd tile sizes, several
heads, random incoming masks and thresholds from -inf to 0 (the same 40
draws on every run: derandomized, so the suite stays deterministic).  For
every draw:
  * mask_out is a subset of mask_in, with no bits past Tk;
  * each output row is library softmax attention (torch SDPA, fp64) over the
    key columns of the tiles that stay live, or 0 if none does;
  * the streaming statistic D_j equals the closed form: the largest rise of a
    row's max in tile j over its max across the live-in tiles before j
    (+inf for the first live-in tile);
  * raising tau can only kill more tiles: live_out(tau_hi) is a subset of
    live_out(tau_lo) for tau_lo <= tau_hi <= 0.
"""
from __future__ import annotations

import math

import numpy as np
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from tests.helpers import bf16_bits, bits_to_f64, sdpa_f64

TAUS = st.one_of(st.just(-math.inf), st.floats(min_value=-12.0, max_value=0.0, allow_nan=False))


@st.composite
def problems(draw):
    N = draw(st.integers(min_value=1, max_value=160))
    d = draw(st.sampled_from([16, 32, 64]))
    Br = draw(st.sampled_from([16, 32, 48, 64]))
    Bc = draw(st.sampled_from([16, 32, 48, 64]))
    H = draw(st.integers(min_value=1, max_value=2))
    scale = draw(st.sampled_from([0.5, 1.0, 2.0, 3.0]))
    seed = draw(st.integers(min_value=0, max_value=10_000))
    live_p = draw(st.sampled_from([1.0, 0.8, 0.5, 0.2]))
    return N, d, Br, Bc, H, scale, seed, live_p


def _inputs(N, d, H, scale, seed):
    g = torch.Generator().manual_seed(seed)
    q = (scale * torch.randn(1, H, N, d, generator=g)).to(torch.bfloat16)
    k = (scale * torch.randn(1, H, N, d, generator=g)).to(torch.bfloat16)
    v = torch.randn(1, H, N, d, generator=g).to(torch.bfloat16)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


def _run(oracle_mod, qkv, N, d, Br, Bc, H, tau, mask_in):
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    items = np.arange(H * Tq)
    return oracle_mod.step(*qkv, B=1, H=H, N=N, d=d, Br=Br, Bc=Bc, tau=tau, items=items, mask_in=mask_in)


@settings(max_examples=40, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(prob=problems(), tau=TAUS, tau2=TAUS)
def test_oracle_properties(oracle_mod, prob, tau, tau2):
    N, d, Br, Bc, H, scale, seed, live_p = prob
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    qkv = _inputs(N, d, H, scale, seed)
    rng = np.random.default_rng(seed)
    live_in = rng.random((H * Tq, Tk)) < live_p
    mask_in = oracle_mod.bool_to_bits(live_in)
    res = _run(oracle_mod, qkv, N, d, Br, Bc, H, tau, mask_in)
    live_out = oracle_mod.bits_to_bool(res["mask_out"], Tk)

    # subset, and no bits past Tk
    assert not (live_out & ~live_in).any()
    if Tk % 32:
        assert not (res["mask_out"][:, W - 1] >> np.uint32(Tk % 32)).any()

    qf, kf, vf = (bits_to_f64(x) for x in qkv)
    logits = np.einsum("bhnd,bhmd->bhnm", qf, kf) / math.sqrt(d)
    for it in range(H * Tq):
        h, i = divmod(it, Tq)
        r0, r1 = i * Br, min(N, (i + 1) * Br)
        cols = np.repeat(live_out[it], Bc)[:N]
        o = res["o"][it, : r1 - r0]
        if not cols.any():
            assert np.all(o == 0.0)
        else:
            ref = sdpa_f64(qf[0, h, r0:r1], kf[0, h], vf[0, h], attn_mask=np.broadcast_to(cols, (r1 - r0, N)).copy())
            assert np.abs(o - ref).max() <= 1e-11 * max(1.0, np.abs(ref).max())
        # closed form of D over the live-in tiles
        s = logits[0, h, r0:r1]
        mloc = np.stack([s[:, j * Bc:min(N, (j + 1) * Bc)].max(axis=1) for j in range(Tk)])
        prefix = None
        for j in range(Tk):
            if not live_in[it, j]:
                assert math.isnan(res["D"][it, j])
                continue
            expect = math.inf if prefix is None else float(np.max(mloc[j] - prefix))
            got = res["D"][it, j]
            assert got == expect if math.isinf(expect) else abs(got - expect) <= 1e-12 * max(1.0, abs(expect))
            if abs(expect - tau) > 1e-9:
                assert live_out[it, j] == (not expect < tau)
            prefix = mloc[j] if prefix is None else np.maximum(prefix, mloc[j])

    # monotone in tau
    lo, hi = min(tau, tau2), max(tau, tau2)
    live_lo = oracle_mod.bits_to_bool(_run(oracle_mod, qkv, N, d, Br, Bc, H, lo, mask_in)["mask_out"], Tk)
    live_hi = oracle_mod.bits_to_bool(_run(oracle_mod, qkv, N, d, Br, Bc, H, hi, mask_in)["mask_out"], Tk)
    assert not (live_hi & ~live_lo).any()
