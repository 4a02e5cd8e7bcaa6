"""The checking build (libsalad_debug.so: every kernel that reads a block mask
checks each row first, SALAD_DEBUG) on the GPU, in a child process that loads
it instead of the release library (debug_child.py says what it checks)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_build_reads_malformed_mask_rows_as_empty_and_reports_them():
    from sparse_linear_hybrid_b200 import build as nvbuild
    lib = nvbuild.build(debug=True)
    env = dict(os.environ, SALAD_LIBRARY=lib)
    res = subprocess.run([sys.executable, os.path.join(HERE, "debug_child.py")], env=env, capture_output=True,
                         text=True, timeout=600)
    print(res.stdout[-4000:], res.stderr[-4000:])
    assert res.returncode == 0
    assert "all checks passed" in res.stdout
