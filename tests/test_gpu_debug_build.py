"""GPU: the checked build (LITE_DEBUG_CHECKS) finds every work item valid on
config 1, edge shapes and imported masks (see tests/debug_build_checks.py)."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_reports_no_bad_work_item():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    res = subprocess.run([sys.executable, "-m", "tests.debug_build_checks"], cwd=ROOT, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-3000:]
    assert "all work items valid" in res.stdout
