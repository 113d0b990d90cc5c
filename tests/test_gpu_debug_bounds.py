"""The bounds-checking debug build of the library (-DDSA_DEBUG_BOUNDS=1):
every kernel checks the indices it is about to use against its buffers and
records a failed check in the status word.  A child process loads that build
(DSA_LIB) and runs every entry point on edge shapes; none may report."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_bounds_build_runs_clean():
    from sparse_attention_token_index_b200 import build as B
    lib = B.build(debug_bounds=True)
    env = dict(os.environ, DSA_LIB=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_cases.py")], env=env, cwd=os.path.dirname(HERE),
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:] + r.stderr[-3000:])
    assert "debug-bounds cases ok" in r.stdout
