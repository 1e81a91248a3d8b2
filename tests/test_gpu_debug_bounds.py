"""The debug bounds-check build on the small cases.

``liblogo_debug.so`` (``make -C token_level_dynamic_seq_b200/csrc debug``) is the
same library with the forward kernels checking every TMA coordinate, gathered
row and stored row against the tensor it addresses before the access (a failed
check is reported by ``logo_check`` as LOGO_ERR_BOUNDS and the access is
skipped).  The small-case parity tests, the caller-list checks and the no-write
canary run against it in a child process (the library is chosen when the
package is first imported): every check must hold, so they pass exactly as
with the normal build.
"""
import ctypes
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG_SO = os.path.join(ROOT, "token_level_dynamic_seq_b200", "liblogo_debug.so")


def test_debug_build_reports_its_flag():
    assert os.path.exists(DEBUG_SO), "build it with: make -C token_level_dynamic_seq_b200/csrc debug"
    lib = ctypes.CDLL(DEBUG_SO)
    lib.logo_build_flags.restype = ctypes.c_uint
    assert lib.logo_build_flags() & 1


def test_small_cases_pass_under_debug_bounds():
    env = dict(os.environ, LOGO_LIBRARY=DEBUG_SO)
    cmd = [sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_parity.py"), "-m", "gpu", "-q", "-x",
           "-p", "no:cacheprovider", "-k", "small_full or named_small or bad_selection or no_writes or running_max"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
