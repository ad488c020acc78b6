"""Pins of the oracle's Newton solve and nonlinear adjoint (torch-sla, technical
summary, "Methodology" 2, nonlinear systems: F(u, theta) = 0, one adjoint solve
J^T lambda = dL/du and one vector-Jacobian product), on the reaction-diffusion
residual F(u) = A u + kappa u^3 - f with A an SPD diffusion matrix, whose
Jacobian A + 3 kappa diag(u^2) is SPD for kappa >= 0.

Pins: a manufactured solution (f built from a chosen u*), the linear special
case kappa = 0, quadratic convergence of the residual norms, and central finite
differences of L = 0.5 ||u - u_obs||^2 in f and kappa through dense Newton.
"""
import numpy as np

from differentiable_sparse_linear_csr_b200 import workloads as W
from oracle import oracle as O


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (d if d > 0 else 1.0)


def _problem(N=12, seed=81, B=None):
    ei, ej = W.grid_edges((N, N))
    n = N * N
    w = W.uniform(seed, W.STREAM_WEIGHTS, ei.shape[0], 0.5, 2.0)
    rp, ci, v = W.weighted_laplacian(n, ei, ej, w, 0.1)
    d = O.diag_positions(rp, ci)
    return n, rp, ci, v, d


def _fns(rp, ci, v, d, kappa, f):
    def residual(U):
        return np.stack([O.spmv(rp, ci, v, u) for u in U]) + kappa * U ** 3 - f

    def jacobian(U):
        J = np.tile(v, (U.shape[0], 1))
        J[:, d] += 3.0 * kappa * U ** 2
        return J
    return residual, jacobian


def test_newton_recovers_a_manufactured_solution():
    n, rp, ci, v, d = _problem()
    us = W.uniform(82, W.STREAM_XSTAR, 2 * n, -2, 2).reshape(2, n)
    kappa = 0.7
    f = np.stack([O.spmv(rp, ci, v, u) for u in us]) + kappa * us ** 3
    res, jac = _fns(rp, ci, v, d, kappa, f)
    u, info = O.newton(rp, ci, res, jac, np.zeros((2, n)), tol=1e-13)
    assert info.converged and info.steps <= 12
    assert rel(u, us) < 1e-12


def test_newton_with_kappa_zero_is_the_linear_solve():
    n, rp, ci, v, d = _problem()
    f = W.normal(83, W.STREAM_B, n)[None, :]
    res, jac = _fns(rp, ci, v, d, 0.0, f)
    u, info = O.newton(rp, ci, res, jac, np.zeros((1, n)), tol=1e-13)
    x, _ = O.pcg(rp, ci, v, f[0], rtol=1e-14)
    assert info.steps == 1 and rel(u[0], x) < 1e-12
    assert rel(u[0], np.linalg.solve(W.csr_to_dense(rp, ci, v), f[0])) < 1e-12


def test_newton_converges_quadratically():
    n, rp, ci, v, d = _problem()
    f = 3.0 * W.normal(84, W.STREAM_B, n)[None, :]
    res, jac = _fns(rp, ci, v, d, 2.0, f)
    _, info = O.newton(rp, ci, res, jac, np.zeros((1, n)), tol=1e-14, max_steps=40)
    r = np.array([x[0] for x in info.residual_norms])
    assert info.converged
    # in the quadratic regime (||F_k|| < 1 here) ||F_{k+1}|| / ||F_k||^2 stays
    # bounded (below 1) while ||F_k|| falls from above 0.1 to 1e-12; under
    # linear convergence that quotient would grow without bound
    tail = [k for k in range(len(r) - 1) if r[k] < 1.0]
    assert len(tail) >= 3 and r[tail[0]] > 0.1
    assert all(r[k + 1] / r[k] ** 2 < 1.0 for k in tail)
    assert r[-1] < 1e-12


def _dense_newton_loss(A, kappa, f, uo):
    u = np.zeros_like(f)
    for _ in range(60):
        F = A @ u + kappa * u ** 3 - f
        J = A + np.diag(3 * kappa * u ** 2)
        du = np.linalg.solve(J, F)
        u = u - du
        if np.linalg.norm(du) < 1e-15 * max(1.0, np.linalg.norm(u)):
            break
    return 0.5 * float(np.sum((u - uo) ** 2)), u


def test_adjoint_gradients_match_central_differences():
    n, rp, ci, v, d = _problem(N=6, seed=85)
    A = W.csr_to_dense(rp, ci, v)
    f = 2.0 * W.normal(85, W.STREAM_B, n)[None, :]
    uo = W.uniform(85, W.STREAM_XSTAR, n, -1, 1)
    kappa = 0.8
    res, jac = _fns(rp, ci, v, d, kappa, f)
    u, info = O.newton(rp, ci, res, jac, np.zeros((1, n)), tol=1e-14)
    assert info.converged
    lam = O.newton_adjoint(rp, ci, jac(u), u - uo)
    # F = A u + kappa u^3 - f:  dF/df = -I, dF/dkappa = u^3
    df = lam[0]                                     # -lambda^T (-I)
    dk = -float(lam[0] @ u[0] ** 3)
    for i in range(n):
        h = 1e-6
        fp, fm = f[0].copy(), f[0].copy()
        fp[i] += h
        fm[i] -= h
        fd = (_dense_newton_loss(A, kappa, fp, uo)[0] - _dense_newton_loss(A, kappa, fm, uo)[0]) / (2 * h)
        assert abs(fd - df[i]) <= 1e-6 * max(abs(fd), 1e-3), (i, fd, df[i])
    h = 1e-6
    fd = (_dense_newton_loss(A, kappa + h, f[0], uo)[0] -
          _dense_newton_loss(A, kappa - h, f[0], uo)[0]) / (2 * h)
    assert abs(fd - dk) <= 1e-6 * max(abs(fd), 1e-3)
