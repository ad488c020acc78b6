"""Pins of the oracle's edge-weighted Laplacian (assembly from edge weights and
the chain rule back to them), against facts fixed outside it.

The operation is the conductivity-to-matrix map of inverse coefficient
learning ("torch-sla: Differentiable Sparse Linear Algebra with Adjoint
Solvers and Sparse Tensor Parallelism for PyTorch", technical summary,
"Experimental results", end-to-end application): A = L_w + shift*I with
A_ij = A_ji = -w_e per edge and A_ii the sum of i's edge weights plus the shift.
Pins: the input generator's own assembly (separate numpy code), exact row sums
and symmetry, central finite differences of the loss through dense solves, the
closed form of the edge gradient, the Euler identity of a map linear in
(w, shift), and hand-built invalid edge lists.
"""
import numpy as np
import pytest

from differentiable_sparse_linear_csr_b200 import workloads as W
from oracle import oracle as O


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (d if d > 0 else 1.0)


def _grid_case(dims, seed, B=None, lo=0.5, hi=2.0):
    ei, ej = W.grid_edges(dims)
    n = int(np.prod(dims))
    m = ei.shape[0]
    w = W.uniform(seed, W.STREAM_WEIGHTS, m * (B or 1), lo, hi)
    return n, ei, ej, (w.reshape(B, m) if B else w)


@pytest.mark.parametrize("case", ["grid2d_batch", "grid3d_lognormal", "knn"])
def test_assembly_matches_the_generators_assembly_bitwise(case):
    if case == "grid2d_batch":
        n, ei, ej, w = _grid_case((8, 8), 4, B=3)
        shift = 1e-2
    elif case == "grid3d_lognormal":
        ei, ej = W.grid_edges((5, 5, 5))
        n = 125
        w = np.exp(W.normal(3, W.STREAM_WEIGHTS, ei.shape[0]))
        shift = 1e-3
    else:
        pts = W.uniform01(5, W.STREAM_POINTS, np.arange(2 * 600, dtype=np.uint64)).reshape(600, 2)
        ei, ej = W.knn_graph_edges(pts, 8)
        n = 600
        w = W.uniform(5, W.STREAM_WEIGHTS, ei.shape[0], 0.5, 2.0)
        shift = 1e-3
    rp, ci, v = W.weighted_laplacian(n, ei, ej, w, shift)
    vo = O.laplacian_assemble(rp, ci, ei, ej, w, shift)
    assert vo.shape == v.shape
    assert np.array_equal(vo.view(np.uint64), np.asarray(v, np.float64).view(np.uint64))


def test_assembly_fp32_equals_fp64_when_every_sum_is_exact():
    # weights k/8 with k <= 16 and a shift of 1/16: every partial sum is a
    # short dyadic number, exact in both precisions
    n, ei, ej, _ = _grid_case((6, 7), 1)
    k = 1 + (np.arange(ei.shape[0]) * 7) % 16
    w = k / 8.0
    rp, ci, _ = W.weighted_laplacian(n, ei, ej, w, 0.0)
    v64 = O.laplacian_assemble(rp, ci, ei, ej, w, 1 / 16)
    v32 = O.laplacian_assemble(rp, ci, ei, ej, w.astype(np.float32), 1 / 16)
    assert v32.dtype == np.float32
    assert np.array_equal(v32.astype(np.float64), v64)


def test_assembly_row_sums_symmetry_and_unnamed_entries():
    n, ei, ej, _ = _grid_case((5, 4), 2)
    w = (1 + np.arange(ei.shape[0]) % 5) / 4.0
    # pattern with two extra symmetric entries (0, 7), (7, 0) that no edge names
    rows = np.concatenate([ei, ej, np.arange(n), [0, 7]])
    cols = np.concatenate([ej, ei, np.arange(n), [7, 0]])
    rp, ci, _, _ = O.coo_to_csr(n, n, rows, cols, np.ones(rows.shape[0]))
    v = O.laplacian_assemble(rp, ci, ei, ej, w, 0.25)
    ones = np.ones(n)
    assert np.array_equal(O.spmv(rp, ci, v, ones), np.full(n, 0.25))   # L_w 1 = 0, exactly
    rpT, ciT, vT, _ = O.transpose(rp, ci, v)
    assert np.array_equal(rpT, rp) and np.array_equal(ciT, ci) and np.array_equal(vT, v)
    s = O.edge_slots(rp, ci, ei, ej)
    extra = [t for t in range(ci.shape[0]) if s.owner[t] < 0 and ci[t] != np.repeat(
        np.arange(n), np.diff(rp))[t]]
    assert len(extra) == 2 and all(v[t] == 0.0 for t in extra)
    assert np.all(v[s.slot_ij] == -w) and np.all(v[s.slot_ji] == -w)


def test_edge_slot_codes():
    # path 0-1-2 with diagonal; pattern of the path graph
    rp = np.array([0, 2, 5, 7], np.int32)
    ci = np.array([0, 1, 0, 1, 2, 1, 2], np.int32)
    ok = O.edge_slots(rp, ci, [0, 1], [1, 2])
    assert ok.code == 0 and ok.where == -1
    assert ok.slot_ij.tolist() == [1, 4] and ok.slot_ji.tolist() == [2, 5]
    assert ok.owner.tolist() == [-1, 0, 0, -1, 1, 1, -1]
    assert (O.edge_slots(rp, ci, [0, 1, 3], [1, 2, 0]).code,
            O.edge_slots(rp, ci, [0, 1, 3], [1, 2, 0]).where) == (1, 2)
    assert (lambda s: (s.code, s.where))(O.edge_slots(rp, ci, [0, -1], [1, 2])) == (1, 1)
    assert (lambda s: (s.code, s.where))(O.edge_slots(rp, ci, [0, 2], [1, 2])) == (2, 1)
    assert (lambda s: (s.code, s.where))(O.edge_slots(rp, ci, [0, 0], [1, 2])) == (3, 1)
    assert (lambda s: (s.code, s.where))(O.edge_slots(rp, ci, [0, 1, 1], [1, 2, 0])) == (4, 2)
    assert (lambda s: (s.code, s.where))(O.edge_slots(rp, ci, [1, 0, 1], [2, 1, 2])) == (4, 2)
    # smallest code wins over a smaller index
    assert (lambda s: (s.code, s.where))(O.edge_slots(rp, ci, [0, 0, 2], [1, 1, 2])) == (2, 2)
    rp_nd = np.array([0, 2, 4, 6], np.int32)                    # row 1 without its diagonal
    ci_nd = np.array([0, 1, 0, 2, 1, 2], np.int32)
    assert (lambda s: (s.code, s.where))(O.edge_slots(rp_nd, ci_nd, [0, 1], [1, 2])) == (5, 1)


def _dense_loss_and_grads(n, ei, ej, w, shift, b, xs):
    rp, ci, v = W.weighted_laplacian(n, ei, ej, w, shift)
    A = W.csr_to_dense(rp, ci, v)
    x = np.linalg.solve(A, b)
    lam = np.linalg.solve(A.T, x - xs)
    return rp, ci, v, x, lam


def _loss(n, ei, ej, w, shift, b, xs):
    rp, ci, v = W.weighted_laplacian(n, ei, ej, w, shift)
    x = np.linalg.solve(W.csr_to_dense(rp, ci, v), b)
    return 0.5 * float(np.sum((x - xs) ** 2))


def test_chain_rule_matches_central_differences():
    n, ei, ej, w = _grid_case((4, 4), 11)
    shift = 0.3
    b = W.uniform(11, W.STREAM_B, n, -1, 1)
    xs = W.uniform(11, W.STREAM_XSTAR, n, -1, 1)
    rp, ci, v, x, lam = _dense_loss_and_grads(n, ei, ej, w, shift, b, xs)
    G = O.grad_values(rp, ci, lam, x)
    dw, ds = O.laplacian_grad_values(rp, ci, ei, ej, G)
    for e in range(ei.shape[0]):
        h = 1e-6 * w[e]
        wp, wm = w.copy(), w.copy()
        wp[e] += h
        wm[e] -= h
        fd = (_loss(n, ei, ej, wp, shift, b, xs) - _loss(n, ei, ej, wm, shift, b, xs)) / (2 * h)
        assert abs(fd - dw[e]) <= 1e-6 * max(abs(fd), 1e-3), (e, fd, dw[e])
    h = 1e-6
    fd = (_loss(n, ei, ej, w, shift + h, b, xs) - _loss(n, ei, ej, w, shift - h, b, xs)) / (2 * h)
    assert abs(fd - ds) <= 1e-6 * max(abs(fd), 1e-3)


def test_chain_rule_closed_form_and_euler_identity():
    # G = -lam x^T on the pattern gives dL/dw_e = (lam_i - lam_j)(x_j - x_i) and
    # dL/dshift = -lam.x; and since A is linear in (w, shift),
    # sum_e w_e dL/dw_e + shift dL/dshift = sum_t vals_t G_t
    n, ei, ej, w = _grid_case((9, 7), 12, B=2)
    shift = 5e-2
    rng_b = W.normal(12, W.STREAM_B, 2 * n).reshape(2, n)
    xs = W.uniform(12, W.STREAM_XSTAR, 2 * n, -1, 1).reshape(2, n)
    rp, ci, v = W.weighted_laplacian(n, ei, ej, w, shift)
    X = np.stack([np.linalg.solve(W.csr_to_dense(rp, ci, v[s]), rng_b[s]) for s in range(2)])
    LAM = np.stack([np.linalg.solve(W.csr_to_dense(rp, ci, v[s]).T, X[s] - xs[s]) for s in range(2)])
    G = O.grad_values(rp, ci, LAM, X)
    dw, ds = O.laplacian_grad_values(rp, ci, ei, ej, G)
    for s in range(2):
        closed = (LAM[s][ei] - LAM[s][ej]) * (X[s][ej] - X[s][ei])
        assert rel(dw[s], closed) < 1e-12
        assert abs(ds[s] + LAM[s] @ X[s]) <= 1e-12 * abs(LAM[s] @ X[s])
        euler = w[s] @ dw[s] + shift * ds[s]
        assert abs(euler - v[s] @ G[s]) <= 1e-12 * abs(v[s] @ G[s])


def test_chain_rule_accumulate_adds():
    n, ei, ej, w = _grid_case((5, 5), 13)
    rp, ci, v = W.weighted_laplacian(n, ei, ej, w, 0.1)
    G = W.uniform(13, W.STREAM_B, ci.shape[0], -1, 1)
    dw0 = W.uniform(13, W.STREAM_XSTAR, ei.shape[0], -1, 1)
    dw, ds = O.laplacian_grad_values(rp, ci, ei, ej, G)
    dwa, dsa = O.laplacian_grad_values(rp, ci, ei, ej, G, dw=dw0, dshift=0.5)
    assert np.array_equal(dwa, dw0 + dw)
    assert dsa == 0.5 + ds
