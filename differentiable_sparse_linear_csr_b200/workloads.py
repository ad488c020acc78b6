"""Seeded synthetic inputs for the sparse SPD solves: patterns, values, right-hand sides.

This module is the only code shared by the CUDA path and the CPU oracle.  It builds
the matrices and vectors that both sides consume and contains none of the solver's
arithmetic (no matrix-vector product, no conjugate-gradient step, no gradient).

Random numbers come from one counter-based generator, SplitMix64 (Steele, Lea and
Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014): the i-th
draw of a stream is the SplitMix64 finaliser applied to ``s0 + (i + 1) * gamma``,
where ``s0`` is derived from the (seed, stream) pair.  Every draw is addressed by
its index, so any element can be regenerated alone and in any order.

Workloads follow the benchmark family of "torch-sla: Differentiable Sparse Linear
Algebra with Adjoint Solvers and Sparse Tensor Parallelism for PyTorch" (technical
summary, "Experimental results": 2-D Poisson, 10^6 DOF, 1000 CG iterations; the
inverse-coefficient-learning application for the batched diffusion case), widened
to a 3-D variable-coefficient diffusion and an unstructured k-nearest-neighbour
graph Laplacian.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream ids of the generator (one per kind of random input).
STREAM_B, STREAM_XSTAR, STREAM_WEIGHTS, STREAM_POINTS = 0, 1, 2, 3


def _finalize(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def _stream_base(seed: int, stream: int) -> np.uint64:
    key = np.array([(int(seed) & 0xFFFFFFFFFFFF) | (int(stream) << 48)], dtype=np.uint64)
    return _finalize(key)[0]


def uniform01(seed: int, stream: int, index: np.ndarray) -> np.ndarray:
    """Uniform draws in [0, 1) with 53 random bits, one per requested index."""
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        ctr = _stream_base(seed, stream) + (idx + np.uint64(1)) * _GAMMA
    u = _finalize(ctr)
    return (u >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def uniform(seed: int, stream: int, count: int, lo: float, hi: float, offset: int = 0) -> np.ndarray:
    u = uniform01(seed, stream, np.arange(offset, offset + count, dtype=np.uint64))
    return lo + (hi - lo) * u


def normal(seed: int, stream: int, count: int, offset: int = 0) -> np.ndarray:
    """Standard normal draws by the Box-Muller transform on index pairs (2i, 2i+1)."""
    i = np.arange(offset, offset + count, dtype=np.uint64)
    u1 = 1.0 - uniform01(seed, stream, 2 * i)          # in (0, 1]
    u2 = uniform01(seed, stream, 2 * i + 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


# ---------------------------------------------------------------------------
# Patterns and values
# ---------------------------------------------------------------------------

def _csr_from_sorted_keys(n: int, rows: np.ndarray, cols: np.ndarray):
    order = np.lexsort((cols, rows))
    rows, cols = rows[order], cols[order]
    counts = np.bincount(rows, minlength=n)
    rowptr = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(counts, out=rowptr[1:])
    return rowptr, cols, order


def poisson1d(N: int):
    """Tridiagonal (-1, 2, -1) on N interior nodes with zero Dirichlet ends."""
    rows, cols, vals = [], [], []
    for i in range(N):
        for j, v in ((i - 1, -1.0), (i, 2.0), (i + 1, -1.0)):
            if 0 <= j < N:
                rows.append(i); cols.append(j); vals.append(v)
    rowptr = np.zeros(N + 1, dtype=np.int32)
    np.cumsum(np.bincount(np.array(rows), minlength=N), out=rowptr[1:])
    return rowptr, np.array(cols, dtype=np.int32), np.array(vals, dtype=np.float64)


def poisson2d(N: int):
    """5-point Laplacian with stencil (4, -1) on an N x N interior grid, Dirichlet zero.

    Unknown (y, x) has index y*N + x.  Boundary neighbours are eliminated, so the
    pattern has 5N^2 - 4N entries.  Entries are exact in binary and the matrix is
    bitwise symmetric.
    """
    idx = np.arange(N * N, dtype=np.int64)
    y, x = idx // N, idx % N
    rows, cols, vals = [], [], []
    for dy, dx, v in ((-1, 0, -1.0), (0, -1, -1.0), (0, 0, 4.0), (0, 1, -1.0), (1, 0, -1.0)):
        ok = (y + dy >= 0) & (y + dy < N) & (x + dx >= 0) & (x + dx < N)
        rows.append(idx[ok]); cols.append((idx + dy * N + dx)[ok]); vals.append(np.full(ok.sum(), v))
    rows, cols, vals = np.concatenate(rows), np.concatenate(cols), np.concatenate(vals)
    rowptr, cols, order = _csr_from_sorted_keys(N * N, rows, cols)
    return rowptr.astype(np.int32), cols.astype(np.int32), vals[order]


def grid_edges(dims):
    """Undirected nearest-neighbour edges (i < j) of a row-major grid, sorted by (i, j)."""
    dims = tuple(int(d) for d in dims)
    n = int(np.prod(dims))
    idx = np.arange(n, dtype=np.int64)
    coords = np.unravel_index(idx, dims)
    strides = [int(np.prod(dims[a + 1:])) for a in range(len(dims))]
    ii, jj = [], []
    for a in range(len(dims)):
        ok = coords[a] + 1 < dims[a]
        ii.append(idx[ok]); jj.append(idx[ok] + strides[a])
    ii, jj = np.concatenate(ii), np.concatenate(jj)
    order = np.lexsort((jj, ii))
    return ii[order], jj[order]


def weighted_laplacian(n: int, ei: np.ndarray, ej: np.ndarray, w: np.ndarray, shift: float):
    """CSR of L_w + shift*I from undirected edges (ei < ej) with weights w.

    A_ij = A_ji = -w_e for edge e = (i, j); A_ii is the sum of the weights of the
    edges at i taken in ascending neighbour index, plus ``shift``.  Every weight is
    stored once per direction, so the result is bitwise symmetric.
    Returns ``rowptr, colind, vals`` with columns sorted within each row.
    """
    w = np.asarray(w, dtype=np.float64)
    nw = w.shape[:-1]                                     # optional batch dims of the weights
    m = ei.shape[0]
    rows = np.concatenate([ei, ej, np.arange(n, dtype=np.int64)])
    cols = np.concatenate([ej, ei, np.arange(n, dtype=np.int64)])
    src = np.concatenate([np.arange(m), np.arange(m), np.full(n, -1)])  # edge id, -1 for diagonal
    rowptr, colind, order = _csr_from_sorted_keys(n, rows, cols)
    src = src[order]
    rows_sorted = rows[order]
    nnz = colind.shape[0]
    wb = w.reshape(-1, m)
    vals = np.empty((wb.shape[0], nnz), dtype=np.float64)
    off = src >= 0
    vals[:, off] = -wb[:, src[off]]
    # Diagonal: weights of row i in ascending neighbour order, then the shift.
    deg = np.diff(rowptr)
    pos_in_row = np.arange(nnz) - rowptr[rows_sorted]
    diag_sum = np.zeros((wb.shape[0], n), dtype=np.float64)
    # Entries of a row sit in ascending column order, so walking the in-row
    # positions k = 0, 1, ... adds each row's weights in ascending neighbour order.
    # A row appears at most once per pass (no repeated fancy indices).
    for k in range(int(deg.max()) if n else 0):
        sel = off & (pos_in_row == k)
        r = rows_sorted[sel]
        diag_sum[:, r] = diag_sum[:, r] + wb[:, src[sel]]
    dpos = np.nonzero(~off)[0]
    vals[:, dpos] = diag_sum[:, rows_sorted[dpos]] + shift
    vals = vals.reshape(nw + (nnz,)) if nw else vals[0]
    return rowptr.astype(np.int32), colind.astype(np.int32), vals


def knn_graph_edges(points: np.ndarray, k: int):
    """Union-symmetrised k-nearest-neighbour graph (self excluded), edges (i<j) sorted."""
    from scipy.spatial import cKDTree
    n = points.shape[0]
    tree = cKDTree(points)
    _, nb = tree.query(points, k=k + 1, workers=-1)
    nb = nb[:, 1:].astype(np.int64)
    i = np.repeat(np.arange(n, dtype=np.int64), k)
    j = nb.reshape(-1)
    lo, hi = np.minimum(i, j), np.maximum(i, j)
    key = np.unique(lo * n + hi)
    return key // n, key % n


def knn_graph_edges_bruteforce(points: np.ndarray, k: int):
    """O(n^2) reference for small point sets; distance ties broken by lower index."""
    n = points.shape[0]
    d2 = ((points[:, None, :] - points[None, :, :]) ** 2).sum(-1)
    np.fill_diagonal(d2, np.inf)
    nb = np.lexsort((np.broadcast_to(np.arange(n), (n, n)), d2), axis=1)[:, :k]
    i = np.repeat(np.arange(n, dtype=np.int64), k)
    j = nb.reshape(-1).astype(np.int64)
    lo, hi = np.minimum(i, j), np.maximum(i, j)
    key = np.unique(lo * n + hi)
    return key // n, key % n


def rcm_permutation(rowptr: np.ndarray, colind: np.ndarray, n: int) -> np.ndarray:
    """Reverse Cuthill-McKee order of a symmetric pattern (new index k holds old perm[k])."""
    import scipy.sparse as sp
    from scipy.sparse.csgraph import reverse_cuthill_mckee
    m = sp.csr_matrix((np.ones(colind.shape[0]), colind, rowptr), shape=(n, n))
    return np.asarray(reverse_cuthill_mckee(m, symmetric_mode=True), dtype=np.int64)


def permute_symmetric(rowptr, colind, vals, perm):
    """P A P^T for new index k = old perm[k]; values moved, never combined."""
    n = rowptr.shape[0] - 1
    inv = np.empty(n, dtype=np.int64)
    inv[perm] = np.arange(n)
    deg = np.diff(rowptr.astype(np.int64))
    new_deg = deg[perm]
    new_rowptr = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(new_deg, out=new_rowptr[1:])
    old_rows = np.repeat(np.arange(n), deg)
    new_rows = inv[old_rows]
    new_cols = inv[colind.astype(np.int64)]
    order = np.lexsort((new_cols, new_rows))
    v = np.asarray(vals)
    return (new_rowptr.astype(np.int32), new_cols[order].astype(np.int32), v[..., order])


def random_spd(n: int, density: float, seed: int, diag_extra: float = 1.0):
    """Small random symmetric, strictly diagonally dominant (hence SPD) matrix in CSR.

    The diagonal varies from row to row, so a Jacobi preconditioner is not a
    multiple of the identity.
    """
    u = uniform01(seed, STREAM_WEIGHTS, np.arange(n * n, dtype=np.uint64)).reshape(n, n)
    mask = np.triu(u < density, 1)
    offv = uniform(seed, STREAM_POINTS, n * n, -1.0, 1.0).reshape(n, n) * mask
    off = offv + offv.T
    dense = off.copy()
    extra = uniform(seed, STREAM_XSTAR, n, 0.0, 3.0, offset=10_000_000)
    dense[np.arange(n), np.arange(n)] = np.abs(off).sum(1) + diag_extra + extra
    return dense_to_csr(dense)


def dense_to_csr(dense: np.ndarray, keep_diagonal: bool = True):
    n_rows, n_cols = dense.shape
    mask = dense != 0
    if keep_diagonal:
        k = min(n_rows, n_cols)
        mask[np.arange(k), np.arange(k)] = True
    rows, cols = np.nonzero(mask)
    rowptr = np.zeros(n_rows + 1, dtype=np.int32)
    np.cumsum(np.bincount(rows, minlength=n_rows), out=rowptr[1:])
    return rowptr, cols.astype(np.int32), dense[rows, cols].astype(np.float64)


def csr_to_dense(rowptr, colind, vals, n_cols=None):
    n = rowptr.shape[0] - 1
    n_cols = n if n_cols is None else n_cols
    d = np.zeros((n, n_cols), dtype=np.float64)
    rows = np.repeat(np.arange(n), np.diff(rowptr.astype(np.int64)))
    np.add.at(d, (rows, colind), vals)
    return d


# ---------------------------------------------------------------------------
# The five benchmark workloads
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    n: int
    rowptr: np.ndarray          # int32 [n+1]
    colind: np.ndarray          # int32 [nnz]
    values: np.ndarray          # float64 [B][nnz]
    b: np.ndarray               # float64 [B][n]
    xstar: np.ndarray           # float64 [B][n]  (target of L = 0.5*||x - x*||^2)
    rtol: float                 # relative residual target (0 when fixed_iters > 0)
    fixed_iters: int            # > 0: run exactly this many iterations
    description: str = ""
    # edge-weighted Laplacians only: the undirected edges (ei, ej) in this
    # workload's row numbering, their weights [B][E] and the diagonal shift
    edges: tuple | None = None
    weights: np.ndarray | None = None
    shift: float = 0.0
    # lists of independent systems only: item s owns rows [item_rows[s], item_rows[s+1])
    item_rows: np.ndarray | None = None

    @property
    def nnz(self) -> int:
        return int(self.colind.shape[0])

    @property
    def batch(self) -> int:
        return int(self.values.shape[0])


def _as_batch(a):
    a = np.asarray(a, dtype=np.float64)
    return a[None, :] if a.ndim == 1 else a


def c1_poisson64(seed: int = 1) -> Workload:
    rp, ci, v = poisson2d(64)
    n = 64 * 64
    return Workload("c1_poisson2d_64", n, rp, ci, _as_batch(v),
                    _as_batch(uniform(seed, STREAM_B, n, -1, 1)),
                    _as_batch(uniform(seed, STREAM_XSTAR, n, -1, 1)),
                    1e-10, 0, "2-D 5-point Dirichlet Poisson 64x64, fp64, PCG to 1e-10")


def c2_poisson1024(seed: int = 2, N: int = 1024, iters: int = 1000) -> Workload:
    rp, ci, v = poisson2d(N)
    n = N * N
    return Workload(f"c2_poisson2d_{N}", n, rp, ci, _as_batch(v),
                    _as_batch(normal(seed, STREAM_B, n)),
                    _as_batch(normal(seed, STREAM_XSTAR, n)),
                    0.0, iters, f"2-D 5-point Poisson {N}x{N}, fixed {iters} forward + {iters} adjoint iterations")


def c3_diffusion3d(seed: int = 3, N: int = 128) -> Workload:
    dims = (N, N, N)
    n = N ** 3
    ei, ej = grid_edges(dims)
    w = np.exp(normal(seed, STREAM_WEIGHTS, ei.shape[0]))
    rp, ci, v = weighted_laplacian(n, ei, ej, w, 1e-3)
    return Workload(f"c3_diffusion3d_{N}", n, rp, ci, _as_batch(v),
                    _as_batch(uniform(seed, STREAM_B, n, -1, 1)),
                    _as_batch(uniform(seed, STREAM_XSTAR, n, -1, 1)),
                    1e-8, 0, f"3-D 7-point log-normal diffusion {N}^3 + 1e-3 I, PCG to 1e-8",
                    (ei, ej), w[None, :], 1e-3)


def c3_batched(seed: int = 3, N: int = 128, B: int = 4) -> Workload:
    """B systems sharing the 3-D 7-point pattern of an N^3 grid, each with its own
    log-normal weights (w = exp(N(0,1)) per edge, system s drawing indices
    [s E, (s+1) E) of the weights stream) + 1e-3 I; b, x* ~ U[-1,1] per system."""
    dims = (N, N, N)
    n = N ** 3
    ei, ej = grid_edges(dims)
    m = ei.shape[0]
    w = np.exp(normal(seed, STREAM_WEIGHTS, B * m)).reshape(B, m)
    rp, ci, v = weighted_laplacian(n, ei, ej, w, 1e-3)
    return Workload(f"c3_batched_{B}x{N}^3", n, rp, ci, v,
                    uniform(seed, STREAM_B, B * n, -1, 1).reshape(B, n),
                    uniform(seed, STREAM_XSTAR, B * n, -1, 1).reshape(B, n),
                    1e-8, 0, f"{B} shared-pattern 3-D 7-point log-normal diffusion systems {N}^3 + 1e-3 I, "
                             f"PCG to 1e-8", (ei, ej), w, 1e-3)


def c4_batched(seed: int = 4, B: int = 1024, N: int = 32) -> Workload:
    n = N * N
    ei, ej = grid_edges((N, N))
    m = ei.shape[0]
    w = uniform(seed, STREAM_WEIGHTS, B * m, 0.5, 2.0).reshape(B, m)
    rp, ci, v = weighted_laplacian(n, ei, ej, w, 1e-2)
    return Workload(f"c4_batched_{B}x{N}x{N}", n, rp, ci, _as_batch(v),
                    normal(seed, STREAM_B, B * n).reshape(B, n),
                    uniform(seed, STREAM_XSTAR, B * n, -1, 1).reshape(B, n),
                    1e-10, 0, f"{B} shared-pattern {N}x{N} diffusion systems + 1e-2 I, PCG to 1e-10",
                    (ei, ej), w, 1e-2)


def list_of_grids(seed: int = 6, B: int = 1024, N_lo: int = 16, N_hi: int = 48) -> Workload:
    """B independent diffusion systems on N_s x N_s grids, N_s uniform in
    [N_lo, N_hi] (sizes from the points stream), each L_w + 1e-2 I with
    w ~ U[0.5, 2] per edge, stored block-diagonally; b ~ N(0,1), x* ~ U[-1,1]."""
    sizes = N_lo + np.floor(uniform01(seed, STREAM_POINTS, np.arange(B, dtype=np.uint64))
                            * (N_hi - N_lo + 1)).astype(np.int64)
    rps, cis, vs, rows, ents, woff = [], [], [], [0], [0], 0
    for N in sizes:
        ei, ej = grid_edges((int(N), int(N)))
        w = uniform(seed, STREAM_WEIGHTS, ei.shape[0], 0.5, 2.0, offset=woff)
        woff += ei.shape[0]
        rp, ci, v = weighted_laplacian(int(N) * int(N), ei, ej, w, 1e-2)
        rps.append(rp[:-1].astype(np.int64) + ents[-1])
        cis.append(ci.astype(np.int64) + rows[-1])
        vs.append(v)
        rows.append(rows[-1] + int(N) * int(N))
        ents.append(ents[-1] + ci.shape[0])
    rowptr = np.concatenate(rps + [np.array([ents[-1]])]).astype(np.int32)
    colind = np.concatenate(cis).astype(np.int32)
    n = rows[-1]
    return Workload(f"list_{B}_grids_{N_lo}to{N_hi}", n, rowptr, colind, np.concatenate(vs)[None, :],
                    _as_batch(normal(seed, STREAM_B, n)), _as_batch(uniform(seed, STREAM_XSTAR, n, -1, 1)),
                    1e-10, 0, f"list of {B} diffusion systems on N x N grids, N uniform in "
                              f"[{N_lo}, {N_hi}], + 1e-2 I, PCG to 1e-10",
                    item_rows=np.array(rows, dtype=np.int32))


def c5_knn(seed: int = 5, npts: int = 8_000_000, k: int = 8, order: str = "generated") -> Workload:
    x = uniform01(seed, STREAM_POINTS, np.arange(2 * npts, dtype=np.uint64)).reshape(npts, 2)
    ei, ej = knn_graph_edges(x, k)
    w = uniform(seed, STREAM_WEIGHTS, ei.shape[0], 0.5, 2.0)
    rp, ci, v = weighted_laplacian(npts, ei, ej, w, 1e-3)
    b = normal(seed, STREAM_B, npts)
    xs = normal(seed, STREAM_XSTAR, npts)
    if order == "rcm":
        perm = rcm_permutation(rp, ci, npts)
        rp, ci, v = permute_symmetric(rp, ci, v, perm)
        b, xs = b[perm], xs[perm]
        inv = np.empty(npts, dtype=np.int64)
        inv[perm] = np.arange(npts)
        ei, ej = inv[ei], inv[ej]                 # the same edges, renumbered
    elif order != "generated":
        raise ValueError(order)
    return Workload(f"c5_knn_{npts}_{order}", npts, rp, ci, _as_batch(v), _as_batch(b), _as_batch(xs),
                    1e-8, 0, f"{k}-NN graph Laplacian on {npts} points ({order} order) + 1e-3 I, PCG to 1e-8",
                    (ei, ej), w[None, :], 1e-3)


CONFIGS = {
    "c1": c1_poisson64,
    "c2": c2_poisson1024,
    "c3": c3_diffusion3d,
    "c4": c4_batched,
    "c5": c5_knn,
}
