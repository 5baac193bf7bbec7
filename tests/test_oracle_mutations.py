"""Mutation check of the oracle's pins (CPU).

Each case plants one plausible mistake in a copy of ``oracle/lite_oracle.c``
(a wrong comparison, sign, index, operand or dropped term), builds the copy
with gcc in a temporary directory and runs the pin suite
(``tests/test_oracle_pins.py``) against it through ``LITE_ORACLE_LIB``.  The
suite must fail on an assertion.  An unmodified copy built and run the same
way must pass, so a failing mutant run means the pins caught the mistake and
not that the harness broke.

Mistakes that cannot change any result are left out on purpose.  One example
is letting a tile killed in this step raise the running max: for tau <= 0 such
a tile never holds a larger row max, so both versions compute the same thing.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lite_oracle.c")

# (name, text in lite_oracle.c, replacement): each text occurs exactly once
MUTANTS = [
    ("tie dies (<= for <)",
     "int dead = (Dj < tau);", "int dead = (Dj <= tau);"),
    ("dead tile keeps its softmax and PV",
     "if (dead) continue;\n                mout_row[j >> 5] |= (1u << (j & 31));",
     "if (!dead) mout_row[j >> 5] |= (1u << (j & 31));"),
    ("rise with the wrong sign",
     "INFINITY : mloc[r] - mrun[r];", "INFINITY : mrun[r] - mloc[r];"),
    ("min over rows instead of max",
     "if (rise > Dj) Dj = rise;", "if (rise < Dj || Dj == -INFINITY) Dj = rise;"),
    ("first processed tile can die",
     "(mrun[r] == -INFINITY) ? INFINITY :", "(mrun[r] == -INFINITY) ? -INFINITY :"),
    ("accumulator rescale dropped",
     "acc[r * d + e] *= alpha;", "acc[r * d + e] *= 1.0;"),
    ("denominator rescale dropped",
     "l[r] = l[r] * alpha + lsum;", "l[r] = l[r] + lsum;"),
    ("scale 1/d instead of 1/sqrt(d)",
     "1.0 / sqrt((double)d)", "1.0 / (double)d"),
    ("V read from K",
     "vt[c * d + e] = bf16_bits_to_double(v[", "vt[c * d + e] = bf16_bits_to_double(k["),
    ("query rows of tile 0 for every tile",
     "q[head_off + (size_t)(r0 + r) * d + e]", "q[head_off + (size_t)r * d + e]"),
    ("last valid key column of a partial tile dropped",
     "(N - c0 < Bc) ? (N - c0) : Bc", "(N - c0 < Bc) ? (N - c0 - 1) : Bc"),
    ("tiles dead on entry processed",
     "if (!((min_row[j >> 5] >> (j & 31)) & 1u)) continue;", "if (0) continue;"),
    ("descending key-tile order",
     "for (int j = 0; j < Tk; ++j) {\n                if (!((min_row",
     "for (int j = Tk - 1; j >= 0; --j) {\n                if (!((min_row"),
    ("mask bit written one place off",
     "mout_row[j >> 5] |= (1u << (j & 31));", "mout_row[j >> 5] |= (1u << ((j + 1) & 31));"),
]


def _build(src_text: str, workdir: str) -> str:
    os.makedirs(workdir, exist_ok=True)
    c = os.path.join(workdir, "lite_oracle.c")
    so = os.path.join(workdir, "liblite_oracle.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", c, "-o", so, "-lm"], check=True)
    return so


def _run_pins(lib_path: str):
    env = dict(os.environ, LITE_ORACLE_LIB=lib_path, OMP_NUM_THREADS="2", CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q", "-rf",
           "-p", "no:cacheprovider", "-m", "not gpu"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout + r.stderr


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = open(SRC).read()
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, f"mutant '{name}': its text must occur exactly once in lite_oracle.c"

    jobs = [("unmodified", src)] + [(name, src.replace(old, new)) for name, old, new in MUTANTS]
    libs = [(name, _build(text, str(tmp_path / f"m{i}"))) for i, (name, text) in enumerate(jobs)]
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda nl: (nl[0],) + _run_pins(nl[1]), libs))

    name0, rc0, out0 = results[0]
    assert rc0 == 0, f"the unmodified copy must pass the pins:\n{out0[-3000:]}"
    survivors = []
    for name, rc, out in results[1:]:
        failed = re.findall(r"^FAILED (\S+)", out, flags=re.M)
        # exit code 1 = tests ran and some failed (not a crash, an import error or a usage error)
        if rc != 1 or not failed:
            survivors.append(f"{name}: rc={rc}\n{out[-1500:]}")
        else:
            print(f"{name}: caught by {failed[0]}")
    assert not survivors, "planted mistakes that no pin caught:\n" + "\n".join(survivors)
