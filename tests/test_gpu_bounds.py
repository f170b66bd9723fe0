"""The whole GPU suite once more against the bounds build of the library
(libm3_bounds.so, loaded under M3_BOUNDS=1): every kernel checks each
global-memory access it makes through a plain pointer against its buffer's
extent, and after every test the suite's own fixture fails the test if any
check failed (m3_stream_status returns M3_ERR_BOUNDS with the site, index and
extent).  The checks record and skip, they never trap, so an index bug shows
up as a failed test with a location instead of a fault.  Runs as a child
process because the library is chosen when it is first loaded."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_gpu_suite_under_device_index_checks():
    from state_space_sequence_ssm_b200 import build
    build.build(bounds=True)
    env = dict(os.environ, M3_BOUNDS="1")
    cmd = [sys.executable, "-m", "pytest", "tests", "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider",
           "--ignore=tests/test_gpu_bounds.py"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout.splitlines()[-1], tail
