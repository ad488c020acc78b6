"""Pins of the oracle's list solve (independent items with their own patterns,
torch-sla's SparseTensorList, technical summary, "Methodology" 1) and of the
list generator.

A list of copies of one pattern must reproduce the shared-pattern batched solve
bit for bit (same arithmetic per item); converged items of mixed sizes must
match dense solves of each item.
"""
import numpy as np

from differentiable_sparse_linear_csr_b200 import workloads as W
from oracle import oracle as O


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def test_list_of_equal_patterns_equals_the_batched_solve():
    w = W.c4_batched(B=5, N=9)
    n, nnz = w.n, w.nnz
    item_rows = np.arange(6) * n
    rowptr = np.concatenate([w.rowptr[:-1] + s * nnz for s in range(5)] + [[5 * nnz]]).astype(np.int32)
    colind = np.concatenate([w.colind + s * n for s in range(5)]).astype(np.int32)
    vals, b = w.values.reshape(-1), w.b.reshape(-1)
    for kw in (dict(rtol=1e-10), dict(fixed_iters=17)):
        x, info = O.pcg_list(item_rows, rowptr, colind, vals, b, **kw)
        xb, ib = O.pcg(w.rowptr, w.colind, w.values, w.b, **kw)
        assert np.array_equal(x.reshape(5, n), xb)
        assert np.array_equal(info.iters, ib.iters) and np.array_equal(info.status, ib.status)
        lam, _ = O.pcg_list(item_rows, rowptr, colind, vals, b, adjoint=True, **kw)
        lb, _ = O.cg_adjoint(w.rowptr, w.colind, w.values, w.b, **kw)
        assert np.array_equal(lam.reshape(5, n), lb)


def test_mixed_size_items_match_dense_solves():
    w = W.list_of_grids(B=7, N_lo=3, N_hi=11)
    ir = w.item_rows
    assert ir[0] == 0 and ir[-1] == w.n and np.all(np.diff(ir) > 0)
    x, info = O.pcg_list(ir, w.rowptr, w.colind, w.values[0], w.b[0], rtol=1e-13)
    assert np.all(info.status == 0) and info.iters.shape == (7,)
    A = W.csr_to_dense(w.rowptr, w.colind, w.values[0])
    for s in range(7):
        o, e = ir[s], ir[s + 1]
        # block-diagonal: nothing couples item s to the others
        assert not A[o:e, :o].any() and not A[o:e, e:].any()
        assert rel(x[o:e], np.linalg.solve(A[o:e, o:e], w.b[0][o:e])) < 1e-11
    # the whole block-diagonal system has the same solution
    assert rel(x, np.linalg.solve(A, w.b[0])) < 1e-11
