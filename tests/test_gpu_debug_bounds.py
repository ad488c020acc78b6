"""The bounds-checking build on the GPU: every solver form, the adjoints, SpMV,
the gradients and the edge-weighted Laplacian run clean (no index out of range)
and match the oracle, and a planted out-of-range column is recorded instead of
read.  The build replaces a memory checker on GPUs where none can run; the
cases run in a separate process that loads libsla_debug_bounds.so."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bounds_checking_build_is_clean_and_matches_the_oracle():
    lib = os.path.join(ROOT, "differentiable_sparse_linear_csr_b200", "libsla_debug_bounds.so")
    assert os.path.exists(lib), "build the bounds-checking library first (__graft_entry__.build())"
    script = os.path.join(ROOT, "tests", "debug_bounds_cases.py")
    r = subprocess.run([sys.executable, script], capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-4000:]
    assert "debug bounds: ok" in r.stdout
