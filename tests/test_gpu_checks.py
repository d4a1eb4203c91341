"""The checked build (-DMOE_CHECKS, libmxfp4_moe_checks.so): parity-green on
good inputs, and a pair id, expert offset or pair_row entry outside its
array sets MOE_DEV_BAD_INDEX instead of addressing memory with it.  Runs in
a child process (MXFP4_MOE_CHECKS=1), because a process loads one library."""
import os
import subprocess
import sys

import pytest

from mxfp4_moe_block_b200 import build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_parity_and_bad_indices():
    build.build(checks=True)
    env = dict(os.environ, MXFP4_MOE_CHECKS="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checks_child.py")],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert r.stdout.strip().splitlines()[-1] == "checks ok"
