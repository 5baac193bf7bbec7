"""Shared test helpers: bf16 marshalling and library reference attention.

Nothing here restates the LiteAttention step; reference values come from
``torch.nn.functional.scaled_dot_product_attention`` (a library routine) or
from plain numpy maxima.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns (same shape)."""
    x = x.detach().to("cpu").contiguous()
    if x.dtype != torch.bfloat16:
        x = x.to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    u = bits.astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def sdpa_f64(q: np.ndarray, k: np.ndarray, v: np.ndarray, attn_mask=None) -> np.ndarray:
    """Library softmax attention in fp64; q [..., Lq, d], k/v [..., Lk, d]; mask True = attend."""
    qt = torch.from_numpy(np.ascontiguousarray(q, dtype=np.float64))
    kt = torch.from_numpy(np.ascontiguousarray(k, dtype=np.float64))
    vt = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64))
    m = None if attn_mask is None else torch.from_numpy(np.ascontiguousarray(attn_mask, dtype=bool))
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m).numpy()


def random_qkv(B, H, N, d, seed, scale_qk=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (scale_qk * torch.randn(B, H, N, d, generator=g)).to(torch.bfloat16)
    k = (scale_qk * torch.randn(B, H, N, d, generator=g)).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


def locality_qkv(B, H, N, d, seed, t=0, device="cuda"):
    """Seeded locality-structured q, k, v of shape [B, H, N, d] (bf16) along a 1-D token line:
    the workloads' generator (q, k = 2 phi + noise, v ~ N(0, 1)) on a (1, 1, N) grid."""
    from temporal_block_sparse_sm_b200 import synthetic
    cfg = synthetic.WorkloadConfig("line", B, H, N, d, d, d, (1, 1, N), t + 1, 0.05, 0.0)
    return synthetic.Workload(cfg, seed=seed, device=device).inputs(t)
