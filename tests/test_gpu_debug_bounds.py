"""The bounds-checking build (libsala_debug.so, SALA_DEBUG_BOUNDS) on the parity suites' small
cases: the same tests, run in a child process with SALA_LIBRARY=debug, must pass -- so no checked
index leaves its buffer on any of them (every test reads the status word, which a failed check
sets to SALA_ERR_BOUNDS) -- and the child must really have loaded the debug build."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _child(args, timeout=900):
    env = dict(os.environ, SALA_LIBRARY="debug")
    return subprocess.run([sys.executable, *args], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=timeout)


def test_child_loads_the_debug_build():
    r = _child(["-c", "from hybrid_sparse_linear_b200 import sala; "
                      "assert sala.debug_bounds_build(); print(sala.LIB_PATH)"])
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().endswith("libsala_debug.so")


def test_parity_suites_pass_under_the_debug_build():
    # small and ragged cases of every kernel family; the full-size and timing-sensitive tests stay
    # with the release build
    r = _child(["-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                "tests/test_gpu_sparse.py", "tests/test_gpu_perhead.py", "tests/test_gpu_linear.py",
                "tests/test_gpu_guards.py", "tests/test_gpu_qknorm.py",
                "-k", "not full_size and not 1m_context and not run_twice and not weak_pilot"])
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-2000:])
