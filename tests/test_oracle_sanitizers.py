"""The float64 oracle built with AddressSanitizer and UndefinedBehaviorSanitizer and
driven through every routine (tests/oracle_sanitize.c): no out-of-bounds access, no
leak, no undefined behaviour. Host-only."""

import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_under_sanitizers():
    if shutil.which("gcc") is None:
        pytest.skip("gcc not installed")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "oracle_sanitize")
        build = subprocess.run(
            ["gcc", "-std=c11", "-O1", "-g", "-pthread", "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
             "-fno-omit-frame-pointer", "-o", exe, os.path.join(ROOT, "tests", "oracle_sanitize.c"),
             os.path.join(ROOT, "oracle", "lq_oracle.c"), "-lm"],
            capture_output=True, text=True)
        if build.returncode != 0 and "sanitize" in build.stderr:
            pytest.skip("sanitizer runtime not available: " + build.stderr.strip().splitlines()[-1])
        assert build.returncode == 0, build.stderr
        env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=1", UBSAN_OPTIONS="halt_on_error=1")
        run = subprocess.run([exe], capture_output=True, text=True, timeout=120, env=env)
        assert run.returncode == 0, run.stdout + run.stderr
        assert "oracle sanitize ok" in run.stdout
