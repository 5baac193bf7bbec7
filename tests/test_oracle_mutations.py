"""Mutation check of the oracle's pins (CPU).

Each case plants one plausible mistake in a copy of one oracle source (a
wrong comparison, sign, index, operand or dropped term), builds the copy with
gcc in a temporary directory and runs that source's pin suite against it
through ``LITE_ORACLE_LIB``: ``tests/test_oracle_pins.py`` for
``oracle/lite_oracle.c`` (the QK-Skip step), ``tests/test_oracle_recall.py``
for ``oracle/recall_oracle.c`` (the fixed-recall step).  The suite must fail
on an assertion.  An unmodified copy built and run the same way must pass, so
a failing mutant run means the pins caught the mistake and not that the
harness broke.

Mistakes that cannot change any result are left out on purpose.  Examples:
letting a tile killed in this step raise the running max (for tau <= 0 such a
tile never holds a larger row max); letting the recall predicate test the
first tile a row processes (its mass bound is infinite, so it is kept
anyway); and ties of the predicates (an exact floating-point tie is not a
case any input reaches on purpose).
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


# the same for recall_oracle.c (the fixed-recall predicate)
RECALL_SRC = os.path.join(ROOT, "oracle", "recall_oracle.c")
RECALL_MUTANTS = [
    ("skipped mass not accumulated",
     "if (mrun[r] != -INFINITY) z[r] += (double)nc * exp(mloc[r] - mrun[r]);", "(void)0;"),
    ("skipped mass not rescaled with the running max",
     "z[r] = z[r] * alpha;", "z[r] = z[r];"),
    ("budget ratio inverted",
     "const double c = (1.0 - p) / p;", "const double c = p / (1.0 - p);"),
    ("full tile width for a partial tile",
     "(double)nc * exp(mloc[r] - mrun[r])) / (c * l[r])", "(double)Bc * exp(mloc[r] - mrun[r])) / (c * l[r])"),
    ("peak weight with the wrong sign",
     "(double)nc * exp(mloc[r] - mrun[r])) / (c * l[r])", "(double)nc * exp(mrun[r] - mloc[r])) / (c * l[r])"),
    ("min over rows instead of max",
     "if (g > Ej) Ej = g;", "if (g < Ej || Ej == -INFINITY) Ej = g;"),
    ("skipped tile keeps its softmax and PV",
     "                    continue;\n                }\n                mout_row[j >> 5] |= (1u << (j & 31));",
     "                }\n                if (!skip) mout_row[j >> 5] |= (1u << (j & 31));"),
    ("budget against kept plus skipped mass",
     "/ (c * l[r]) - 1.0;", "/ (c * (l[r] + z[r])) - 1.0;"),
    ("V read from K",
     "vt[cc * d + e] = rc_bf16_to_double(v[", "vt[cc * d + e] = rc_bf16_to_double(k["),
]


def _build(src_text: str, workdir: str, which: str = "lite") -> str:
    """One mutated oracle source with the other one unmodified, as one library."""
    import oracle
    os.makedirs(workdir, exist_ok=True)
    name = "lite_oracle.c" if which == "lite" else "recall_oracle.c"
    c = os.path.join(workdir, name)
    with open(c, "w") as f:
        f.write(src_text)
    other = RECALL_SRC if which == "lite" else SRC
    return oracle.compile_library([c, other], os.path.join(workdir, "liblite_oracle.so"))


def _run_pins(lib_path: str, pins: str = "tests/test_oracle_pins.py"):
    env = dict(os.environ, LITE_ORACLE_LIB=lib_path, OMP_NUM_THREADS="2", CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "pytest", pins, "-x", "-q", "-rf",
           "-p", "no:cacheprovider", "-m", "not gpu"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout + r.stderr


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("which", ["lite", "recall"])
def test_every_planted_mistake_fails_a_pin(tmp_path, which):
    path, mutants, pins = ((SRC, MUTANTS, "tests/test_oracle_pins.py") if which == "lite" else
                           (RECALL_SRC, RECALL_MUTANTS, "tests/test_oracle_recall.py"))
    src = open(path).read()
    for name, old, new in mutants:
        assert src.count(old) == 1, f"mutant '{name}': its text must occur exactly once in {os.path.basename(path)}"

    jobs = [("unmodified", src)] + [(name, src.replace(old, new)) for name, old, new in mutants]
    libs = [(name, _build(text, str(tmp_path / f"m{i}"), which)) for i, (name, text) in enumerate(jobs)]
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda nl: (nl[0],) + _run_pins(nl[1], pins), libs))

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
