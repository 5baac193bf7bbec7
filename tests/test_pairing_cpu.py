"""The pairing of query tiles into work items (host logic, CPU).

``pair_tiles`` in ``csrc/liteattn_internal.cuh`` is compiled for the host with
g++ and must agree with the rule stated in ``tests/pairing.py``: every query
tile in exactly one pair, ceil(Tq/2) pairs, and adjacent tiles for stride 1.
"""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

from tests.pairing import pairs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "temporal_block_sparse_sm_b200", "csrc")

PROBE = r"""
#include <cstdio>
#define __host__
#define __device__
#define __forceinline__ inline
#include "liteattn_internal.cuh"
int main() {
    for (int Tq = 1; Tq <= 130; ++Tq)
        for (int s = 1; s <= 33; ++s)
            for (int p = 0; p < (Tq + 1) / 2; ++p) {
                int a, b;
                lite::pair_tiles(p, Tq, s, a, b);
                printf("%d %d %d %d %d\n", Tq, s, p, a, b);
            }
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_pair_tiles_follows_the_rule(tmp_path):
    src = tmp_path / "probe.cpp"
    src.write_text(PROBE)
    exe = tmp_path / "probe"
    subprocess.run(["g++", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {}
    for line in out:
        if line.strip():
            Tq, s, p, a, b = map(int, line.split())
            got.setdefault((Tq, s), []).append((a, b))
    assert len(got) == 130 * 33
    for (Tq, s), lst in got.items():
        assert lst == pairs(Tq, s), (Tq, s)


@pytest.mark.parametrize("Tq", [1, 2, 7, 64, 255, 256, 844])
@pytest.mark.parametrize("s", [1, 2, 12, 28])
def test_rule_covers_every_tile_once(Tq, s):
    ps = pairs(Tq, s)
    assert len(ps) == (Tq + 1) // 2
    tiles = [t for a, b in ps for t in (a, b) if t >= 0]
    assert sorted(tiles) == list(range(Tq))
    if s == 1:
        assert ps == [(2 * p, 2 * p + 1 if 2 * p + 1 < Tq else -1) for p in range((Tq + 1) // 2)]
