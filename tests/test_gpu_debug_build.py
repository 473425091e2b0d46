"""The debug build of the library (libhstu_debug.so, compiled with
-DHSTU_DEBUG): the attention kernels check the row and column indices of their
direct global accesses and report a failed check as HSTU_DEVICE_BOUNDS in the
device status word, skipping the access instead of trapping.  The checks run
in a child process that loads the debug build (HSTU_DEBUG_BUILD=1): valid
inputs match the oracle with no report; rows past the declared row count are
reported (all of that case's buffers hold the rows, so nothing outside an
allocation is touched)."""
import os
import subprocess
import sys

import pytest

from hstu_sequential_transducer_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_bounds_checks():
    build.build(debug=True)
    env = dict(os.environ, HSTU_DEBUG_BUILD="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_child.py")],
                       capture_output=True, text=True, timeout=900, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "debug build ok" in r.stdout
