"""The parity tests of the core path, rerun in a child process against the
bounds-checked build of the library (libgs_checked.so, loaded with
GS_CHECKED=1): on valid inputs every device-side check must pass (the
session's status word stays 0) and every result must still match the
oracle. No input here is out of range on purpose: out-of-range arguments are
covered by the host-side validation tests."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_core_parity_under_the_checked_build():
    env = dict(os.environ, GS_CHECKED="1")
    files = ["tests/test_gpu_parity.py", "tests/test_gpu_binning.py", "tests/test_gpu_hit_bits.py",
             "tests/test_gpu_async.py", "tests/test_gpu_multiview.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-s", *files], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=1200)
    tail = r.stdout[-4000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert "checked build: device-side check status 0" in r.stdout, tail
