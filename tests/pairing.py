"""The query-tile pairing rule of the library's work items, stated for the tests.

Tiles go in blocks of 2s (s = the plan's pair stride); within a block tile r
pairs with tile r + s; a last, shorter block of m tiles pairs r with r +
ceil(m/2).  s = 1 gives adjacent pairs (2p, 2p + 1).
"""
from __future__ import annotations


def pairs(Tq: int, s: int = 1):
    """[(tile_a, tile_b or -1)] for pairs 0 .. ceil(Tq/2) - 1."""
    out = []
    base = 0
    while base < Tq:
        m = min(2 * s, Tq - base)
        h = (m + 1) // 2
        for r in range(h):
            out.append((base + r, base + r + h if r + h < m else -1))
        base += m
    return out
