"""Checks of the seeded input generators (no solver arithmetic here)."""
import numpy as np
import pytest

from differentiable_sparse_linear_csr_b200 import workloads as W


def test_splitmix_is_counter_based_and_uniform():
    a = W.uniform01(7, 0, np.arange(100_000, dtype=np.uint64))
    b = W.uniform01(7, 0, np.arange(50_000, 100_000, dtype=np.uint64))
    assert np.array_equal(a[50_000:], b)                 # any index regenerates alone
    assert a.min() >= 0.0 and a.max() < 1.0
    assert abs(a.mean() - 0.5) < 0.005 and abs(a.var() - 1 / 12) < 0.002
    c = W.uniform01(7, 1, np.arange(100_000, dtype=np.uint64))
    assert abs(np.corrcoef(a, c)[0, 1]) < 0.02          # streams are independent
    z = W.normal(3, 0, 200_000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    # first SplitMix64 outputs for state 0 (published test vector of the generator)
    g = np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        out = W._finalize(np.array([g, g * np.uint64(2)], dtype=np.uint64))
    assert [int(v) for v in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4]


@pytest.mark.parametrize("N", [1, 2, 5, 64])
def test_poisson2d_nnz_closed_form(N):
    rp, ci, v = W.poisson2d(N)
    assert ci.shape[0] == 5 * N * N - 4 * N
    assert rp[-1] == ci.shape[0]
    assert set(np.unique(v).tolist()) <= {-1.0, 4.0}


@pytest.mark.parametrize("N", [2, 3, 8])
def test_grid3d_laplacian_nnz_closed_form(N):
    ei, ej = W.grid_edges((N, N, N))
    assert ei.shape[0] == 3 * N * N * (N - 1)
    rp, ci, v = W.weighted_laplacian(N ** 3, ei, ej, np.ones(ei.shape[0]), 1e-3)
    assert ci.shape[0] == 7 * N ** 3 - 6 * N ** 2
    d = W.csr_to_dense(rp, ci, v)
    assert np.array_equal(d, d.T)
    assert np.allclose(d.sum(1), 1e-3)                   # Laplacian rows sum to the shift


def test_c4_shapes_and_ranges():
    w = W.c4_batched(B=8)
    assert w.values.shape == (8, 4992) and w.b.shape == (8, 1024)
    rows = np.repeat(np.arange(w.n), np.diff(w.rowptr))
    off = rows != w.colind
    assert np.all(-w.values[:, off] >= 0.5) and np.all(-w.values[:, off] <= 2.0)
    for s in range(8):
        d = W.csr_to_dense(w.rowptr, w.colind, w.values[s])
        assert np.array_equal(d, d.T)
        assert np.all(np.linalg.eigvalsh(d) > 0)


def test_knn_graph_against_brute_force():
    pts = W.uniform01(5, W.STREAM_POINTS, np.arange(2 * 2000, dtype=np.uint64)).reshape(2000, 2)
    ei, ej = W.knn_graph_edges(pts, 8)
    bi, bj = W.knn_graph_edges_bruteforce(pts, 8)
    assert np.array_equal(ei, bi) and np.array_equal(ej, bj)
    rp, ci, v = W.weighted_laplacian(2000, ei, ej, W.uniform(5, W.STREAM_WEIGHTS, ei.shape[0], 0.5, 2), 1e-3)
    deg = np.diff(rp)
    assert deg.min() >= 9                                 # 8 neighbours + diagonal at least


def test_rcm_is_a_bandwidth_reducing_permutation():
    w = W.c5_knn(npts=5000)
    r = W.c5_knn(npts=5000, order="rcm")
    perm = W.rcm_permutation(w.rowptr, w.colind, w.n)
    assert np.array_equal(np.sort(perm), np.arange(w.n))

    def bandwidth(rp, ci):
        rows = np.repeat(np.arange(rp.shape[0] - 1), np.diff(rp))
        return int(np.abs(rows - ci).max())

    assert bandwidth(r.rowptr, r.colind) < bandwidth(w.rowptr, w.colind)
    assert r.nnz == w.nnz
    d0 = W.csr_to_dense(w.rowptr, w.colind, w.values[0])
    d1 = W.csr_to_dense(r.rowptr, r.colind, r.values[0])
    assert np.array_equal(d1, d0[np.ix_(perm, perm)])     # P A P^T, values moved not combined
    assert np.array_equal(r.b[0], w.b[0][perm])


@pytest.mark.parametrize("make", [lambda: W.c4_batched(B=3, N=8), lambda: W.c3_diffusion3d(N=6),
                                  lambda: W.c5_knn(npts=2000), lambda: W.c5_knn(npts=2000, order="rcm")])
def test_edge_weighted_workloads_carry_their_edges(make):
    """Edges, weights and shift reproduce the workload's values through the
    oracle's assembly bit for bit.  In RCM order the workload's values are the
    generated-order matrix permuted, whose diagonals were summed in the old
    neighbour order, while assembly from the renumbered edges sums them in the
    new order: off-diagonal entries still agree bit for bit, diagonals to
    rounding."""
    from oracle import oracle as O
    w = make()
    ei, ej = w.edges
    assert ei.shape == ej.shape and w.weights.shape == (w.batch, ei.shape[0])
    v = O.laplacian_assemble(w.rowptr, w.colind, ei, ej, w.weights, w.shift).reshape(w.values.shape)
    if "rcm" not in w.name:
        assert np.array_equal(v.view(np.uint64), w.values.view(np.uint64))
        return
    d = O.diag_positions(w.rowptr, w.colind)
    off = np.ones(w.nnz, bool)
    off[d] = False
    assert np.array_equal(v[:, off], w.values[:, off])
    assert np.all(np.abs(v[:, d] - w.values[:, d]) <= 32 * 2.0 ** -52 * np.abs(w.values[:, d]))
