"""The GPU suite once more against the bounds-checking build of the library
(libquarot_dbg.so, compiled with QUAROT_DEBUG_BOUNDS): there every kernel
checks, before each global store of an output, that the bytes lie inside that
output, skips the store and records QUAROT_ERR_DEVICE_BOUNDS if not.  Every
test of the suite asserts a clean device status after its calls, so a green
run means no kernel computed an out-of-range output address on any of the
suite's shapes (ragged tiles, odd head counts, the full-size launches), and
that the checks change no result.  Run as a child process, because the
binding picks the library when it is imported."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_gpu_suite_under_bounds_checking_build():
    import __graft_entry__
    __graft_entry__.build()
    env = dict(os.environ, QUAROT_DEBUG_BOUNDS="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests"), "--ignore", os.path.join(ROOT, "tests", "test_gpu_debug_bounds.py")]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in tail
