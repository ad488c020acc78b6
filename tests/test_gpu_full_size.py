"""Full-size workloads: the GPU path against the CPU oracle at the sizes and in
the launch configuration the benchmark times.

Element by element against the oracle, solution, adjoint and value gradient:
the 1024x1024 Poisson system at its fixed 1000 + 1000 iterations (fp64 and
fp32); the 3-D diffusion at fixed counts and in the benchmark's tolerance mode
at the GPU's own iteration counts (fp64 and fp32); every system of the batch;
the kNN graph in both orders at a fixed count.  Besides, properties that hold
at any size, computed with scipy from the GPU's outputs (true residual, adjoint
and Euler identities, the gradient formula on sampled entries), for the
tolerance-mode runs.  The oracle never receives a GPU result as input: where it
runs the GPU's iteration count, it starts from the same inputs and iterates on
its own.
"""
import numpy as np
import pytest
import scipy.sparse as sp
import torch

import differentiable_sparse_linear_csr_b200 as sla
from differentiable_sparse_linear_csr_b200 import _lib as L
from differentiable_sparse_linear_csr_b200 import workloads as W
from oracle import oracle as O

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = torch.device("cuda:0")
TOL_X64, TOL_G64, TOL_X32 = 1e-8, 1e-6, 1e-4


def T(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def H(t):
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()


def rel(a, ref):
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(a - ref) / np.linalg.norm(ref))


def _pipeline(A, vals, b, xs, **opts):
    """Forward solve, g = x - x*, adjoint solve, value gradient (GPU)."""
    x, fi = A.cg(vals, b, **opts)
    g = x - xs
    lam, ai = A.cg(vals, g, adjoint=True, **opts)
    G = A.grad_values(lam, x)
    return x, lam, G, fi, ai


@pytest.mark.parametrize("dtype", [torch.float64, torch.float32])
def test_c2_poisson1024_fixed_1000_elementwise(dtype):
    w = W.c2_poisson1024()
    npdt = np.float64 if dtype == torch.float64 else np.float32
    v, b, xs = w.values.astype(npdt), w.b.astype(npdt), w.xstar.astype(npdt)
    xo, io = O.pcg(w.rowptr, w.colind, v[0], b[0], fixed_iters=1000)
    lo, _ = O.cg_adjoint(w.rowptr, w.colind, v[0], (xo - xs[0]).astype(npdt), fixed_iters=1000)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    A = sla.CSR(T(w.rowptr), T(w.colind), dtype=dtype, symmetric=True)
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), fixed_iters=1000)
    assert H(fi.iters)[0] == 1000 and H(ai.iters)[0] == 1000
    assert H(fi.status)[0] == L.SLA_FIXED_DONE
    if dtype == torch.float64:
        assert rel(H(x)[0], xo) < TOL_X64
        assert rel(H(lam)[0], lo) < TOL_G64
        assert rel(H(G)[0], Go) < TOL_G64
    else:
        assert rel(H(x)[0], xo) < TOL_X32
        assert rel(H(lam)[0], lo) < TOL_X32
        assert rel(H(G)[0], Go) < TOL_X32


def _properties(w, x, lam, G, rtol, b, xs, vals):
    """Checks that hold for any converged solve, at any size (scipy, float64)."""
    A = sp.csr_matrix((vals.astype(np.float64), w.colind, w.rowptr), shape=(w.n, w.n))
    x64, l64, b64 = x.astype(np.float64), lam.astype(np.float64), b.astype(np.float64)
    g = x64 - xs.astype(np.float64)
    # true residuals of both solves (recursive residual <= rtol; drift is small)
    assert np.linalg.norm(b64 - A @ x64) <= 1.5 * rtol * np.linalg.norm(b64)
    assert np.linalg.norm(g - A.T @ l64) <= 1.5 * rtol * np.linalg.norm(g)
    # g.x = lambda.b for symmetric A: with r_x = b - A x and r_l = g - A lambda,
    # g.x - lambda.b = r_l.x - lambda.r_x, bounded by the residuals
    rx = np.linalg.norm(b64 - A @ x64)
    rl = np.linalg.norm(g - A.T @ l64)
    assert abs(g @ x64 - l64 @ b64) <= 1.01 * (rl * np.linalg.norm(x64) + rx * np.linalg.norm(l64)) + 1e-300
    # Euler: sum_t G_t v_t = -lambda.(A x)
    assert abs(G.astype(np.float64) @ vals.astype(np.float64) + l64 @ (A @ x64)) <= \
        1e-10 * np.abs(G.astype(np.float64) * vals).sum()
    # the gradient formula, entry by entry on a sample (exact: one product each)
    rows = np.repeat(np.arange(w.n), np.diff(w.rowptr))
    idx = np.random.default_rng(0).integers(0, w.nnz, 20000)
    assert np.array_equal(G[idx], -(lam[rows[idx]] * x[w.colind[idx]]))


def test_c3_diffusion3d_fixed_and_tolerance():
    w = W.c3_diffusion3d()
    A = sla.CSR(T(w.rowptr), T(w.colind), symmetric=True)
    v, b, xs = w.values, w.b, w.xstar
    # element by element at a fixed count
    k = 100
    xo, _ = O.pcg(w.rowptr, w.colind, v[0], b[0], fixed_iters=k)
    lo, _ = O.cg_adjoint(w.rowptr, w.colind, v[0], xo - xs[0], fixed_iters=k)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), fixed_iters=k)
    assert rel(H(x)[0], xo) < TOL_X64
    assert rel(H(lam)[0], lo) < TOL_G64
    assert rel(H(G)[0], Go) < TOL_G64
    # the benchmark's tolerance mode: properties, and the oracle's iteration count
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), rtol=1e-8)
    assert H(fi.status)[0] == L.SLA_CONVERGED and H(ai.status)[0] == L.SLA_CONVERGED
    _, io = O.pcg(w.rowptr, w.colind, v[0], b[0], rtol=1e-8)
    assert abs(int(H(fi.iters)[0]) - int(io.iters[0])) <= max(2, 0.01 * io.iters[0])
    _properties(w, H(x)[0], H(lam)[0], H(G)[0], 1e-8, b[0], xs[0], v[0])


def test_c3_diffusion3d_tolerance_mode_elementwise_at_the_gpu_counts():
    """The benchmark's run (PCG to 1e-8, adjoint to 1e-8, gradient), element by
    element: the oracle runs exactly the GPU's forward and adjoint iteration
    counts (the reading for ties at the tolerance) on its own iterates."""
    w = W.c3_diffusion3d()
    A = sla.CSR(T(w.rowptr), T(w.colind), symmetric=True)
    v, b, xs = w.values, w.b, w.xstar
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), rtol=1e-8)
    kf, ka = int(H(fi.iters)[0]), int(H(ai.iters)[0])
    assert H(fi.status)[0] == L.SLA_CONVERGED and H(ai.status)[0] == L.SLA_CONVERGED
    xo, _ = O.pcg(w.rowptr, w.colind, v[0], b[0], fixed_iters=kf)
    lo, _ = O.cg_adjoint(w.rowptr, w.colind, v[0], xo - xs[0], fixed_iters=ka)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    assert rel(H(x)[0], xo) < TOL_X64
    assert rel(H(lam)[0], lo) < TOL_G64
    assert rel(H(G)[0], Go) < TOL_G64


def test_c3_diffusion3d_fp32_forward_adjoint_gradient():
    """fp32 at a fixed 200 + 200 iterations against the fp32 oracle: solution,
    adjoint and value gradient element by element at the fp32 bar."""
    w = W.c3_diffusion3d()
    A = sla.CSR(T(w.rowptr), T(w.colind), dtype=torch.float32, symmetric=True)
    v, b, xs = (w.values.astype(np.float32), w.b.astype(np.float32), w.xstar.astype(np.float32))
    k = 200
    xo, _ = O.pcg(w.rowptr, w.colind, v[0], b[0], fixed_iters=k)
    lo, _ = O.cg_adjoint(w.rowptr, w.colind, v[0], (xo - xs[0]).astype(np.float32), fixed_iters=k)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), fixed_iters=k)
    assert H(fi.iters)[0] == k and H(ai.iters)[0] == k
    assert rel(H(x)[0], xo) < TOL_X32
    assert rel(H(lam)[0], lo) < TOL_X32
    assert rel(H(G)[0], Go) < TOL_X32
    # the benchmark's fp32 run (tolerance 1e-8 on the recursive residual), at
    # the GPU's own counts on the oracle's side
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), rtol=1e-8)
    kf, ka = int(H(fi.iters)[0]), int(H(ai.iters)[0])
    assert H(fi.status)[0] == L.SLA_CONVERGED and H(ai.status)[0] == L.SLA_CONVERGED
    assert kf < 5000 and ka < 5000
    xo, _ = O.pcg(w.rowptr, w.colind, v[0], b[0], fixed_iters=kf)
    lo, _ = O.cg_adjoint(w.rowptr, w.colind, v[0], (xo - xs[0]).astype(np.float32), fixed_iters=ka)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    assert rel(H(x)[0], xo) < TOL_X32
    assert rel(H(lam)[0], lo) < TOL_X32
    assert rel(H(G)[0], Go) < TOL_X32


def test_c4_batched_all_systems():
    w = W.c4_batched()
    A = sla.CSR(T(w.rowptr), T(w.colind), batch=w.batch, symmetric=True)
    v, b, xs = w.values, w.b, w.xstar
    k = 60
    xo, _ = O.pcg(w.rowptr, w.colind, v, b, fixed_iters=k)
    lo, _ = O.cg_adjoint(w.rowptr, w.colind, v, xo - xs, fixed_iters=k)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), fixed_iters=k)
    assert max(rel(H(x)[s], xo[s]) for s in range(w.batch)) < TOL_X64
    assert max(rel(H(lam)[s], lo[s]) for s in range(w.batch)) < TOL_G64
    assert max(rel(H(G)[s], Go[s]) for s in range(w.batch)) < TOL_G64
    # tolerance mode: every system converges, counts agree with the oracle's
    x, fi = A.cg(T(v), T(b), rtol=1e-10)
    _, io = O.pcg(w.rowptr, w.colind, v, b, rtol=1e-10)
    assert np.all(H(fi.status) == L.SLA_CONVERGED)
    assert np.all(np.abs(H(fi.iters) - io.iters) <= np.maximum(2, 0.01 * io.iters))


@pytest.mark.parametrize("order", ["generated", "rcm"])
def test_c5_knn_fixed_and_tolerance(order):
    w = W.c5_knn(order=order)
    A = sla.CSR(T(w.rowptr), T(w.colind), symmetric=True)
    v, b, xs = w.values, w.b, w.xstar
    # forward, adjoint and value gradient element by element at a fixed count
    k = 20
    xo, _ = O.pcg(w.rowptr, w.colind, v[0], b[0], fixed_iters=k)
    lo, _ = O.cg_adjoint(w.rowptr, w.colind, v[0], xo - xs[0], fixed_iters=k)
    Go = O.grad_values(w.rowptr, w.colind, lo, xo)
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), fixed_iters=k)
    assert H(fi.iters)[0] == k and H(ai.iters)[0] == k
    assert rel(H(x)[0], xo) < TOL_X64
    assert rel(H(lam)[0], lo) < TOL_G64
    assert rel(H(G)[0], Go) < TOL_G64
    # the benchmark's tolerance mode: properties at full size
    x, lam, G, fi, ai = _pipeline(A, T(v), T(b), T(xs), rtol=1e-8)
    assert H(fi.status)[0] == L.SLA_CONVERGED and H(ai.status)[0] == L.SLA_CONVERGED
    _properties(w, H(x)[0], H(lam)[0], H(G)[0], 1e-8, b[0], xs[0], v[0])
