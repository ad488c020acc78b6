"""GPU interleaved batch solver (values [entry][system], vectors [row][system];
batches of 2 and 4 systems sharing a pattern) against the CPU oracle's batched
PCG on the same seeded inputs, and against the batch-major grid solver.

The on-chip grid variant is turned off so that these small systems take the
path that large batches take.  Tolerances as for the other solvers: fp64 x
1e-8, fp32 x 1e-4, gradients 1e-6; at a fixed count iterations and statuses
are equal.
"""
import numpy as np
import pytest
import torch

import differentiable_sparse_linear_csr_b200 as sla
from differentiable_sparse_linear_csr_b200 import _lib as L
from differentiable_sparse_linear_csr_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
GRID = L.SLA_STRATEGY_GRID


def T(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def H(t):
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()


def rel(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    d = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / (d if d > 0 else 1.0))


def _cases(B):
    yield W.c3_batched(N=13, B=B)                 # 2197 rows, log-normal weights
    w = W.c4_batched(B=B, N=37)                   # 1369 rows, ragged against any tile
    yield w


def _make(w, dtype, monkeypatch, interleave="1"):
    monkeypatch.setenv("SLA_GRID_ONCHIP", "0")
    monkeypatch.setenv("SLA_INTERLEAVE", interleave)
    return sla.CSR(T(w.rowptr), T(w.colind), batch=w.batch, dtype=dtype, symmetric=True)


@pytest.mark.parametrize("B", [2, 4])
@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_fixed_iterations_parity(B, dtype, monkeypatch):
    npdt = np.float64 if dtype == torch.float64 else np.float32
    tol = 1e-8 if dtype == torch.float64 else 1e-4
    for w in _cases(B):
        A = _make(w, dtype, monkeypatch)
        assert A.props.interleaved == 1
        v, b = w.values.astype(npdt), w.b.astype(npdt)
        for k in (1, 7, 60):
            x, info = A.cg(T(v), T(b), fixed_iters=k, strategy=GRID)
            xo, io = O.pcg(w.rowptr, w.colind, v, b, fixed_iters=k)
            assert np.array_equal(H(info.iters), io.iters) and np.array_equal(H(info.status), io.status)
            for s in range(B):
                assert rel(H(x)[s], xo[s]) < tol, (w.name, k, s)


@pytest.mark.parametrize("B", [2, 4])
def test_tolerance_mode_and_agreement_with_the_batch_major_solver(B, monkeypatch):
    for w in _cases(B):
        A = _make(w, torch.float64, monkeypatch)
        x, info = A.cg(T(w.values), T(w.b), rtol=1e-10, strategy=GRID)
        _, io = O.pcg(w.rowptr, w.colind, w.values, w.b, rtol=1e-10)
        it = H(info.iters)
        assert np.all(H(info.status) == 0) and np.all(H(info.relres) <= 1e-10)
        assert np.all(np.abs(it - io.iters) <= np.maximum(2, 0.01 * io.iters))
        for s in range(B):
            xo, _ = O.pcg(w.rowptr, w.colind, w.values[s], w.b[s], fixed_iters=int(it[s]))
            assert rel(H(x)[s], xo) < 1e-8
        Ab = _make(w, torch.float64, monkeypatch, interleave="0")
        assert Ab.props.interleaved == 0
        xb, ib = Ab.cg(T(w.values), T(w.b), rtol=1e-10, strategy=GRID)
        assert np.all(np.abs(H(ib.iters) - it) <= 2)
        assert max(rel(H(xb)[s], H(x)[s]) for s in range(B)) < 1e-8


def test_systems_stop_on_their_own(monkeypatch):
    """System 0 has b = 0, system 1 a NaN, system 2 an initial guess, system 3
    a tight cap: each reports what the oracle reports for it alone."""
    w = W.c3_batched(N=11, B=4)
    b = w.b.copy()
    b[0] = 0.0
    b[1, 5] = np.nan
    x0 = np.zeros_like(b)
    x0[2] = W.uniform(5, 1, w.n, -1, 1)
    A = _make(w, torch.float64, monkeypatch)
    x, info = A.cg(T(w.values), T(b), rtol=1e-10, max_iter=25, x0=T(x0), strategy=GRID)
    st, it = H(info.status), H(info.iters)
    for s in range(4):
        xo, io = O.pcg(w.rowptr, w.colind, w.values[s], b[s], rtol=1e-10, max_iter=25, x0=x0[s])
        assert st[s] == io.status[0] and it[s] == io.iters[0], s
        if s != 1:
            assert rel(H(x)[s], xo) < 1e-8, s
    assert st[0] == L.SLA_CONVERGED and it[0] == 0 and not H(x)[0].any()
    assert st[1] == L.SLA_NONFINITE


def test_adjoint_through_autograd(monkeypatch):
    w = W.c3_batched(N=12, B=4)
    A = _make(w, torch.float64, monkeypatch)
    vt = T(w.values).requires_grad_(True)
    bt = T(w.b).requires_grad_(True)
    x = A.solve(vt, bt, rtol=1e-12, strategy=GRID)
    (0.5 * ((x - T(w.xstar)) ** 2).sum()).backward()
    xo, _ = O.pcg(w.rowptr, w.colind, w.values, w.b, rtol=1e-12)
    lo, _ = O.cg_adjoint(w.rowptr, w.colind, w.values, xo - w.xstar, rtol=1e-12)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    for s in range(4):
        assert rel(H(x)[s], xo[s]) < 1e-8
        assert rel(H(bt.grad)[s], lo[s]) < 1e-6
        assert rel(H(vt.grad)[s], Go[s]) < 1e-6


def test_bounded_wait_times_out_without_hanging(monkeypatch):
    w = W.c3_batched(N=16, B=2)
    A = _make(w, torch.float64, monkeypatch)
    _, info = A.cg(T(w.values), T(w.b), fixed_iters=500, strategy=GRID, wait_timeout_ns=1)
    assert np.all(H(info.status) == L.SLA_TIMED_OUT)
    x, info = A.cg(T(w.values), T(w.b), fixed_iters=20, strategy=GRID)
    xo, _ = O.pcg(w.rowptr, w.colind, w.values, w.b, fixed_iters=20)
    assert np.all(H(info.status) == L.SLA_FIXED_DONE)
    assert max(rel(H(x)[s], xo[s]) for s in range(2)) < 1e-8


@pytest.mark.parametrize("B", [2, 4])
@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_row_ahead_column_loads_are_bit_identical(B, dtype, monkeypatch):
    """Uniform 7-wide slices with 16-bit columns: loading the next row's column
    offsets ahead changes no result bit."""
    npdt = np.float64 if dtype == torch.float64 else np.float32
    w = W.c3_batched(N=32, B=B)
    A = _make(w, dtype, monkeypatch)
    assert A.props.interleaved == 1 and A.props.sliced == 2 and A.props.sliced_col_bytes == 2
    v, b = T(w.values.astype(npdt)), T(w.b.astype(npdt))
    out = {}
    for pipe in ("1", "0"):
        monkeypatch.setenv("SLA_SELL_PIPE", pipe)
        out[pipe], _ = A.cg(v, b, fixed_iters=40, strategy=GRID)
    assert torch.equal(out["1"], out["0"])
    xo, _ = O.pcg(w.rowptr, w.colind, w.values.astype(npdt), w.b.astype(npdt), fixed_iters=40)
    tol = 1e-8 if dtype == torch.float64 else 1e-4
    for s in range(B):
        assert rel(H(out["1"])[s], xo[s]) < tol


def test_fp64_batches_default_to_batch_major(monkeypatch):
    monkeypatch.setenv("SLA_GRID_ONCHIP", "0")
    monkeypatch.delenv("SLA_INTERLEAVE", raising=False)
    w = W.c3_batched(N=13, B=2)
    A64 = sla.CSR(T(w.rowptr), T(w.colind), batch=2, dtype=torch.float64, symmetric=True)
    A32 = sla.CSR(T(w.rowptr), T(w.colind), batch=2, dtype=torch.float32, symmetric=True)
    assert A64.props.interleaved == 0 and A32.props.interleaved == 1
