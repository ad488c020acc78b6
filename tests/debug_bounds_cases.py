"""Solver and kernel cases under the bounds-checking build (run as a script).

Loads libsla_debug_bounds.so (SLA_LIBRARY_VARIANT=debug_bounds), in which every
index a kernel takes from the pattern, and every shared-memory or cluster-rank
index derived from one, is checked before use and recorded instead of used when
out of range.  Runs every solver form on small systems (thread-block cluster,
block per system with and without the matrix in shared memory, persistent grid
with vectors on chip or in HBM, tile flags or a third barrier, sliced (uniform or
per-slice widths, rows sorted within windows, 16- or 32-bit columns) or CSR
rows, two-barrier form, the
interleaved batch, rows loading their column offsets a row ahead, lists of
systems, the allocation-free entry point), the
adjoints (symmetric and through A^T's pattern), SpMV both ways, both value
gradients and the edge-weighted Laplacian; compares each result with the CPU
oracle and requires a clean bounds record.  Then plants one out-of-range
column in a pattern created without validation and requires the record to
name it (the kernels read x[0] in its place and do not fault).  Prints
"debug bounds: ok" when every check holds.
"""
import os
import sys

os.environ["SLA_LIBRARY_VARIANT"] = "debug_bounds"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np   # noqa: E402
import torch         # noqa: E402

import differentiable_sparse_linear_csr_b200 as sla          # noqa: E402
from differentiable_sparse_linear_csr_b200 import _lib as L   # noqa: E402
from differentiable_sparse_linear_csr_b200 import workloads as W  # noqa: E402
from oracle import oracle as O   # noqa: E402

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


def clean(label):
    torch.cuda.synchronize()
    v, code, idx = L.sla_debug_bounds_report()
    assert v == 0, f"{label}: {v} out-of-range indices, first code {code} index {idx}"
    print(f"{label}: ok")


def pipeline(label, rp, ci, v, b, xs, tol_x=1e-8, tol_g=1e-6, env=None, symmetric=True, **opts):
    """Forward, adjoint and value gradient against the oracle at a fixed count."""
    for k, val in (env or {}).items():
        os.environ[k] = val
    try:
        B = v.shape[0]
        A = sla.CSR(T(rp), T(ci), batch=B, symmetric=symmetric)
        x, _ = A.cg(T(v), T(b), **opts)
        lam, _ = A.cg(T(v), x - T(xs), adjoint=True, **opts)
        G = A.grad_values(lam, x)
    finally:
        for k in (env or {}):
            os.environ.pop(k, None)
    k = opts["fixed_iters"]
    xo, _ = O.pcg(rp, ci, v, b, fixed_iters=k)
    lo, _ = O.cg_adjoint(rp, ci, v, xo - xs, fixed_iters=k)
    Go = O.grad_values(rp, ci, lo, xo)
    for s in range(B):
        assert rel(H(x)[s], xo[s]) < tol_x, (label, s)
        assert rel(H(lam)[s], lo[s]) < tol_g, (label, s)
        assert rel(H(G)[s], Go[s]) < tol_g, (label, s)
    clean(label)


def main():
    assert "bounds-checking" in L.sla_version(), L.sla_version()
    L.sla_debug_bounds_report(reset=True)
    w = W.c1_poisson64()
    pipeline("c1 cluster", w.rowptr, w.colind, w.values, w.b, w.xstar, fixed_iters=60,
             strategy=L.SLA_STRATEGY_CLUSTER)
    pipeline("c1 block", w.rowptr, w.colind, w.values, w.b, w.xstar, fixed_iters=60,
             strategy=L.SLA_STRATEGY_BLOCK)
    w = W.c4_batched(B=24, N=16)
    pipeline("batch block, matrix in shared memory", w.rowptr, w.colind, w.values, w.b, w.xstar,
             fixed_iters=40, strategy=L.SLA_STRATEGY_BLOCK)
    pipeline("batch block, matrix through L2", w.rowptr, w.colind, w.values, w.b, w.xstar,
             fixed_iters=40, strategy=L.SLA_STRATEGY_BLOCK, env={"SLA_BLOCK_RESIDENT": "0"})
    pipeline("batch grid", w.rowptr, w.colind, w.values, w.b, w.xstar, fixed_iters=40,
             strategy=L.SLA_STRATEGY_GRID)
    w = W.c3_diffusion3d(N=40)
    for label, env in (("3-D grid on chip, two barriers", {}),
                       ("3-D grid on chip, three barriers", {"SLA_GRID2": "0"}),
                       ("3-D grid, HBM, per-slice widths", {"SLA_GRID_ONCHIP": "0", "SLA_SELL_UNIFORM": "0"}),
                       ("3-D grid, vectors in HBM, sliced", {"SLA_GRID_ONCHIP": "0"}),
                       ("3-D grid, vectors in HBM, CSR rows", {"SLA_GRID_ONCHIP": "0", "SLA_SELL": "0"}),
                       ("3-D grid, HBM, 32-bit columns", {"SLA_GRID_ONCHIP": "0", "SLA_SELL_D16": "0"}),
                       ("3-D grid on chip, three barriers, no tile flags", {"SLA_GRID2": "0",
                                                                           "SLA_TILE_FLAGS": "0"})):
        pipeline(label, w.rowptr, w.colind, w.values, w.b, w.xstar, fixed_iters=30,
                 strategy=L.SLA_STRATEGY_GRID, env=env)
    rp, ci, v = W.random_spd(12000, 0.0005, 9, diag_extra=0.3)   # irregular rows: sorted windows
    pipeline("irregular rows, vectors in HBM, sorted windows", rp, ci, v[None, :],
             W.uniform(8, 0, 12000, -1, 1)[None, :], W.uniform(8, 1, 12000, -1, 1)[None, :], fixed_iters=30,
             strategy=L.SLA_STRATEGY_GRID, env={"SLA_GRID_ONCHIP": "0"})
    w = W.c3_batched(N=32, B=2)   # uniform 7-wide slices: columns loaded a row ahead
    pipeline("interleaved batch of 2", w.rowptr, w.colind, w.values, w.b, w.xstar, fixed_iters=30,
             strategy=L.SLA_STRATEGY_GRID, env={"SLA_GRID_ONCHIP": "0", "SLA_INTERLEAVE": "1"})
    pipeline("interleaved batch of 2, per-slice widths", w.rowptr, w.colind, w.values, w.b, w.xstar,
             fixed_iters=30, strategy=L.SLA_STRATEGY_GRID,
             env={"SLA_GRID_ONCHIP": "0", "SLA_INTERLEAVE": "1", "SLA_SELL_UNIFORM": "0"})
    pipeline("batch of 2 in HBM, batch-major", w.rowptr, w.colind, w.values, w.b, w.xstar, fixed_iters=30,
             strategy=L.SLA_STRATEGY_GRID, env={"SLA_GRID_ONCHIP": "0", "SLA_INTERLEAVE": "0"})
    # one 2-D grid on chip with uniform 5-wide slices (columns loaded a row ahead), three
    # phases with tile flags and the two-barrier form
    rp, ci, v = W.poisson2d(100)
    b2, x2 = W.uniform(12, 0, 10000, -1, 1)[None, :], W.uniform(12, 1, 10000, -1, 1)[None, :]
    for label, env in (("2-D grid on chip, three phases", {"SLA_GRID2": "0"}),
                       ("2-D grid on chip, two barriers", {"SLA_GRID2": "2"})):
        pipeline(label, rp, ci, v[None, :], b2, x2, fixed_iters=30, strategy=L.SLA_STRATEGY_GRID, env=env)
    # a non-symmetric pattern: adjoint and SpMV through A^T's pattern
    rp, ci, v = W.random_spd(1500, 0.004, 5, diag_extra=0.5)
    pipeline("adjoint through the transposed pattern", rp, ci, v[None, :], W.normal(5, 0, 1500)[None, :],
             W.uniform(5, 1, 1500, -1, 1)[None, :], symmetric=False, fixed_iters=25)
    A = sla.CSR(T(rp), T(ci), symmetric=False)
    x = W.uniform(6, 0, 1500, -1, 1)
    assert rel(H(A.spmv(T(v), T(x), transpose=True)), O.spmv(*O.transpose(rp, ci, v, 1500)[:3], x)) < 1e-14
    assert np.array_equal(H(A.matvec_grad_values(T(x), T(x)))[0], -O.grad_values(rp, ci, x, x))
    clean("SpMV and gradients")
    # lists of systems
    items = [W.poisson2d(m)[:2] for m in (5, 9, 14)]
    Ls = sla.CSRList.from_items(items, symmetric=True, device=DEV)
    vals = np.concatenate([W.poisson2d(m)[2] for m in (5, 9, 14)])
    bl = W.normal(7, 0, int(Ls.n_rows))
    xl, _ = Ls.cg(T(vals), T(bl), fixed_iters=10)
    xo, _ = O.pcg_list(H(Ls.item_rows), H(Ls.rowptr), H(Ls.colind), vals, bl, fixed_iters=10)
    assert rel(H(xl).ravel(), xo) < 1e-8
    clean("list of systems")
    # the allocation-free entry point
    rp, ci, v = W.poisson2d(60)
    b = W.normal(8, 0, 3600)
    x = torch.empty(1, 3600, dtype=torch.float64, device=DEV)
    L.sla_cg_solve_noalloc(3600, ci.shape[0], T(rp), T(ci), 1, L.SLA_F64, T(v[None, :]), T(b[None, :]), x,
                           L.make_opts(fixed_iters=20, strategy=L.SLA_STRATEGY_GRID), L.make_info())
    assert rel(H(x)[0], O.pcg(rp, ci, v, b, fixed_iters=20)[0]) < 1e-8
    clean("allocation-free solve")
    # the edge-weighted Laplacian
    ei, ej = W.grid_edges((12, 12))
    wts = W.uniform(9, W.STREAM_WEIGHTS, ei.shape[0], 0.5, 2.0)
    rp, ci, v = W.weighted_laplacian(144, ei, ej, wts, 0.1)
    A = sla.CSR(T(rp), T(ci), symmetric=True)
    E = sla.EdgeLaplacian(A, T(ei.astype(np.int32)), T(ej.astype(np.int32)))
    vals = H(E.assemble_values(T(wts), 0.1))
    assert np.array_equal(vals[0], O.laplacian_assemble(rp, ci, ei, ej, wts, 0.1))
    lam, xx = W.uniform(10, 0, 144, -1, 1), W.uniform(10, 1, 144, -1, 1)
    dw, ds = E.grad(T(lam), T(xx))
    dwo, _ = O.laplacian_grad_values(rp, ci, ei, ej, O.grad_values(rp, ci, lam, xx))
    assert np.array_equal(H(dw)[0], dwo)
    clean("edge-weighted Laplacian")

    # a column index out of range, planted in a pattern created without validation:
    # the kernels record it and read x[0] in its place
    n_rows, n_cols = 3000, 2500
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 8, n_rows)
    cols = [np.sort(rng.choice(n_cols, k, replace=False)) for k in lens]
    bad_row = n_rows - 1
    cols[bad_row][-1] = n_cols + 5            # rows stay sorted: it is the row's last entry
    rp = np.zeros(n_rows + 1, np.int32)
    np.cumsum(lens, out=rp[1:])
    ci = np.concatenate(cols).astype(np.int32)
    A = sla.CSR(T(rp), T(ci), n_cols=n_cols, symmetric=False, validate=False)
    v = W.uniform(11, 0, ci.shape[0], -1, 1)
    x = W.uniform(11, 1, n_cols, -1, 1)
    y = H(A.spmv(T(v), T(x)))[0]
    n_bad, code, idx = L.sla_debug_bounds_report(reset=True)
    assert n_bad >= 1 and code == 1 and idx == n_cols + 5, (n_bad, code, idx)
    ok_rows = np.arange(n_rows - 1)
    y_ok = O.spmv(rp[:n_rows], ci[:rp[n_rows - 1]], v[:rp[n_rows - 1]], x)
    assert rel(y[ok_rows], y_ok) < 1e-14
    clean("after reset")
    print("debug bounds: ok")


if __name__ == "__main__":
    main()
