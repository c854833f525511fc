"""The bounds-checking debug build (FFD_DEBUG) stands in for a memory
sanitizer: every global index the decode kernel computes is checked against
the extent the shape implies, and a violation sets FFD_DEVICE_FLAG_BOUNDS
instead of trapping.  The small parity cases of both key formats, the pseudo
maximum and the fused append run on it with no flag raised and the oracle's
results (debug_bounds_run.py, in its own process: a process loads one of the two
libraries)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_build_raises_no_bounds_flag_on_the_parity_cases():
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_run.py")],
                       capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "no flags" in r.stdout
