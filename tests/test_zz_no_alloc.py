"""The allocation-free solve against the regular solve, through the C ABI.

sla_cg_solve_noalloc serves callers that may not allocate device memory while
they solve (runtimes that reserve all device memory up front, loops that cannot
afford an allocation's implicit synchronisation, plugins that must not use their
host's allocator): it keeps its scratch in the library's static device array.
Two calls in a row must both match sla_cg_solve, which shows that what the first
call leaves in the shared array does not leak into the second.  This file is
collected last so that a run stopping at the first failure has run every other
test before it.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from differentiable_sparse_linear_csr_b200 import _lib as L
from differentiable_sparse_linear_csr_b200 import workloads as W
import differentiable_sparse_linear_csr_b200 as sla

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL_X64, TOL_X32 = 1e-8, 1e-4


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _info(B):
    return [torch.full((B,), -7, dtype=torch.int32, device=DEV),
            torch.zeros(B, dtype=torch.float64, device=DEV),
            torch.full((B,), -7, dtype=torch.int32, device=DEV)]


@pytest.mark.parametrize("case", ["poisson_fixed", "batched_tolerance", "fp32"])
def test_noalloc_matches_regular_solve_twice(case, monkeypatch):
    # the reference handle runs the same grid variant (vectors in global memory)
    monkeypatch.setenv("SLA_GRID_ONCHIP", "0")
    if case == "batched_tolerance":
        w = W.c4_batched(B=6, N=20)
        rp, ci, v, b = w.rowptr, w.colind, w.values, w.b
        opts = L.make_opts(rtol=1e-10, strategy=L.SLA_STRATEGY_GRID)
        dt, tol = torch.float64, TOL_X64
    else:
        rp, ci, v = W.poisson2d(150)
        b = W.normal(3, W.STREAM_B, 150 * 150)[None, :]
        v = v[None, :]
        opts = L.make_opts(fixed_iters=120, strategy=L.SLA_STRATEGY_GRID)
        dt = torch.float32 if case == "fp32" else torch.float64
        tol = TOL_X32 if case == "fp32" else TOL_X64
    B, n, nnz = v.shape[0], rp.shape[0] - 1, ci.shape[0]
    rpt = torch.from_numpy(rp).to(DEV)
    cit = torch.from_numpy(ci).to(DEV)
    vt = torch.from_numpy(v).to(DEV, dt).contiguous()
    bt = torch.from_numpy(b).to(DEV, dt).contiguous()
    # the existing entry point, with a caller workspace
    A = sla.CSR(rpt, cit, batch=B, dtype=dt, symmetric=True)
    x_ref = torch.empty(B, n, dtype=dt, device=DEV)
    ref_info = _info(B)
    ws = torch.empty(L.sla_workspace_bytes(A.handle, L.SLA_OP_CG), dtype=torch.uint8, device=DEV)
    L.sla_cg_solve(A.handle, vt, bt, x_ref, opts, L.make_info(*ref_info), ws)
    for call in range(2):
        x = torch.full((B, n), float("nan"), dtype=dt, device=DEV)
        info = _info(B)
        L.sla_cg_solve_noalloc(n, nnz, rpt, cit, B, L.dtype_code(dt), vt, bt, x, opts,
                               L.make_info(*info))
        torch.cuda.synchronize()
        assert torch.equal(info[2], ref_info[2]), call
        assert torch.equal(info[0], ref_info[0]), call
        for s in range(B):
            assert _rel(x[s], x_ref[s]) < tol, (call, s)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    n = 1_000_000                                 # 36 MB of fp64 scratch > 16 MiB
    rp = torch.arange(n + 1, dtype=torch.int32, device=DEV)
    ci = torch.arange(n, dtype=torch.int32, device=DEV)
    v = torch.ones(n, dtype=torch.float64, device=DEV)
    b = torch.ones(n, dtype=torch.float64, device=DEV)
    x = torch.empty(n, dtype=torch.float64, device=DEV)
    with pytest.raises(L.SlaError, match="built-in limit"):
        L.sla_cg_solve_noalloc(n, n, rp, ci, 1, L.SLA_F64, v, b, x, L.make_opts(), L.make_info())


def test_noalloc_follows_the_current_context():
    """A caller that manages its own contexts (the driver API's, or the device
    after a reset) gets the scratch array of the context it calls from: in the
    primary context, in two created contexts and back, two allocation-free
    calls in a row match sla_cg_solve.  Runs as a separate process that makes
    no PyTorch CUDA calls, so the contexts are the script's own."""
    script = os.path.join(os.path.dirname(os.path.abspath(__file__)), "noalloc_contexts.py")
    r = subprocess.run([sys.executable, script], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "noalloc contexts: ok" in r.stdout
