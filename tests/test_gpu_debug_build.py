"""The debug build (liblq_debug.so, -DLQ_DEBUG: device-side bounds checks that
skip an out-of-range access and report LQ_ERR_BOUNDS) on the GPU: every entry
point on small cases against the oracle with no check failing, and the
reporting path through its self-test. The library is chosen when the package
is imported, so the run is a child process with LQ_DEBUG=1."""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_debug_build_parity_and_bounds_selftest():
    env = dict(os.environ, LQ_DEBUG="1")
    env.pop("LQ_FAULT", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_run.py")], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "debug build ok" in r.stdout
