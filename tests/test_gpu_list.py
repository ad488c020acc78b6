"""GPU list solve (independent items with their own patterns, torch-sla's
SparseTensorList, technical summary, "Methodology" 1) against the oracle's
per-item solves on the same seeded inputs.

Tolerances as for the shared-pattern solver: fp64 x 1e-8, fp32 x 1e-4,
gradients 1e-6; iteration counts and statuses at a fixed count are equal.
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


def T(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def H(t):
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()


def rel(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    d = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / (d if d > 0 else 1.0))


def _with_big_item(w_small, N_big=80, seed=7):
    """Append one N_big x N_big item, larger than a block's shared memory."""
    ei, ej = W.grid_edges((N_big, N_big))
    wts = W.uniform(seed, W.STREAM_WEIGHTS, ei.shape[0], 0.5, 2.0)
    rp, ci, v = W.weighted_laplacian(N_big * N_big, ei, ej, wts, 1e-2)
    n0, e0 = w_small.n, w_small.nnz
    rowptr = np.concatenate([w_small.rowptr[:-1], rp.astype(np.int64) + e0]).astype(np.int32)
    colind = np.concatenate([w_small.colind, ci + n0]).astype(np.int32)
    vals = np.concatenate([w_small.values[0], v])
    n = n0 + N_big * N_big
    b = np.concatenate([w_small.b[0], W.normal(seed, W.STREAM_B, N_big * N_big)])
    item_rows = np.concatenate([w_small.item_rows, [n]]).astype(np.int32)
    return item_rows, rowptr, colind, vals, b


def _make(item_rows, rowptr, colind, dtype=torch.float64, symmetric=True):
    return sla.CSRList(T(item_rows), T(rowptr), T(colind), dtype=dtype, symmetric=symmetric)


@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_fixed_iterations_parity_with_an_item_beyond_shared_memory(dtype):
    npdt = np.float64 if dtype == torch.float64 else np.float32
    tol = 1e-8 if dtype == torch.float64 else 1e-4
    # 5 vectors of the big item exceed a block's shared memory in either precision
    N_big = 80 if dtype == torch.float64 else 120
    item_rows, rowptr, colind, vals, b = _with_big_item(W.list_of_grids(B=40, N_lo=4, N_hi=40), N_big)
    A = _make(item_rows, rowptr, colind, dtype)
    p = A.props
    assert p.n_items == 41 and p.item_rows_max == N_big ** 2 and p.item_smem_rows < N_big ** 2
    v, bb = vals.astype(npdt), b.astype(npdt)
    for k in (1, 7, 60):
        x, info = A.cg(T(v), T(bb), fixed_iters=k)
        xo, io = O.pcg_list(item_rows, rowptr, colind, v, bb, fixed_iters=k)
        assert np.array_equal(H(info.iters), io.iters) and np.array_equal(H(info.status), io.status)
        xg = H(x).reshape(-1)
        for s in range(41):
            o, e = item_rows[s], item_rows[s + 1]
            assert rel(xg[o:e], xo[o:e]) < tol, (k, s)


def test_tolerance_mode_per_item_and_reproducible():
    w = W.list_of_grids(B=64, N_lo=4, N_hi=48)
    A = _make(w.item_rows, w.rowptr, w.colind)
    x, info = A.cg(T(w.values[0]), T(w.b[0]), rtol=1e-10)
    it = H(info.iters)
    _, io = O.pcg_list(w.item_rows, w.rowptr, w.colind, w.values[0], w.b[0], rtol=1e-10)
    assert np.all(H(info.status) == 0) and np.all(H(info.relres) <= 1e-10)
    assert np.all(np.abs(it - io.iters) <= np.maximum(2, 0.01 * io.iters))
    # iterates agree with the oracle's at the GPU's per-item counts
    for s in range(64):
        o, e = w.item_rows[s], w.item_rows[s + 1]
        rp = (w.rowptr[o:e + 1] - w.rowptr[o]).astype(np.int32)
        ci = (w.colind[w.rowptr[o]:w.rowptr[e]] - o).astype(np.int32)
        xo, _ = O.pcg(rp, ci, w.values[0][w.rowptr[o]:w.rowptr[e]], w.b[0][o:e], fixed_iters=int(it[s]))
        assert rel(H(x).reshape(-1)[o:e], xo) < 1e-8
    x2, _ = A.cg(T(w.values[0]), T(w.b[0]), rtol=1e-10)
    assert np.array_equal(H(x), H(x2))


def test_items_report_their_own_outcomes():
    """One item with a NaN right-hand side, one indefinite, one with b = 0: the
    others converge as if alone."""
    w = W.list_of_grids(B=6, N_lo=5, N_hi=9)
    ir = w.item_rows
    v, b = w.values[0].copy(), w.b[0].copy()
    b[ir[1] + 2] = np.nan                                  # item 1: non-finite
    t0, t1 = w.rowptr[ir[3]], w.rowptr[ir[4]]
    v[t0:t1] = -v[t0:t1]                                   # item 3: negative diagonal
    b[ir[4]:ir[5]] = 0.0                                   # item 4: zero rhs
    A = _make(ir, w.rowptr, w.colind)
    x, info = A.cg(T(v), T(b), rtol=1e-10)
    xo, io = O.pcg_list(ir, w.rowptr, w.colind, v, b, rtol=1e-10)
    st = H(info.status)
    assert st.tolist() == io.status.tolist()
    assert st[1] == L.SLA_NONFINITE and st[3] == L.SLA_BREAKDOWN and st[4] == L.SLA_CONVERGED
    assert H(info.iters)[4] == 0 and not H(x).reshape(-1)[ir[4]:ir[5]].any()
    for s in (0, 2, 5):
        o, e = ir[s], ir[s + 1]
        assert st[s] == 0 and rel(H(x).reshape(-1)[o:e], xo[o:e]) < 1e-8


@pytest.mark.parametrize("symmetric", [True, False])
def test_solve_backward_matches_the_oracle(symmetric):
    """Autograd through CSRList.solve: one adjoint solve per item (on the
    transposed pattern when the handle is not flagged symmetric) and the value
    gradient -lambda_i x_j on the block-diagonal pattern."""
    w = W.list_of_grids(B=12, N_lo=4, N_hi=30)
    A = _make(w.item_rows, w.rowptr, w.colind, symmetric=symmetric)
    vt = T(w.values[0]).requires_grad_(True)
    bt = T(w.b[0]).requires_grad_(True)
    x = A.solve(vt, bt, rtol=1e-12)
    (0.5 * ((x - T(w.xstar[0])) ** 2).sum()).backward()
    xo, _ = O.pcg_list(w.item_rows, w.rowptr, w.colind, w.values[0], w.b[0], rtol=1e-12)
    lo, _ = O.pcg_list(w.item_rows, w.rowptr, w.colind, w.values[0], xo - w.xstar[0], adjoint=True,
                       rtol=1e-12)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    assert rel(H(x), xo) < 1e-8
    assert rel(H(bt.grad), lo) < 1e-6
    assert rel(H(vt.grad), Go) < 1e-6
    assert H(A.last_adjoint_info.status).shape == (12,)


def test_block_structure_is_checked():
    w = W.list_of_grids(B=3, N_lo=3, N_hi=4)
    ci = w.colind.copy()
    t = w.rowptr[w.item_rows[1]]                           # first entry of item 1
    ci[t] = 0                                              # a column of item 0
    rp = w.rowptr
    # keep the row's columns increasing so only the block rule fails
    row = w.item_rows[1]
    ci[rp[row]:rp[row + 1]] = np.sort(ci[rp[row]:rp[row + 1]])
    with pytest.raises(L.SlaError, match="block"):
        _make(w.item_rows, rp, ci)
    with pytest.raises(L.SlaError):
        _make(np.array([0, 5, 3, w.n], np.int32), w.rowptr, w.colind)
    with pytest.raises(L.SlaError):
        A = _make(w.item_rows, w.rowptr, w.colind)
        A.cg(T(w.values[0]), T(w.b[0]), strategy=L.SLA_STRATEGY_GRID)
