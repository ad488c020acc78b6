"""GPU Newton solve and nonlinear adjoint against the oracle (torch-sla,
technical summary, "Methodology" 2, nonlinear systems).

Residual F(u; w, kappa, f) = A(w) u + kappa u^3 - f with A(w) the
edge-weighted Laplacian plus a shift (assembled by EdgeLaplacian, applied by
CSR.matvec, both differentiable), Jacobian A(w) + 3 kappa diag(u^2).  The
gradients in w, kappa and f come from one adjoint solve and one vector-Jacobian
product through autograd; the oracle gives the same from its Newton iteration,
its adjoint solve, its value gradient and its chain rule to edge weights.
"""
import numpy as np
import pytest
import torch

import differentiable_sparse_linear_csr_b200 as sla
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


def test_newton_solve_and_its_adjoint_match_the_oracle():
    N, B, shift = 24, 2, 0.1
    n = N * N
    ei, ej = W.grid_edges((N, N))
    w = W.uniform(91, W.STREAM_WEIGHTS, B * ei.shape[0], 0.5, 2.0).reshape(B, -1)
    kappa = np.array([0.6])
    f = 2.0 * W.normal(91, W.STREAM_B, B * n).reshape(B, n)
    uo = W.uniform(91, W.STREAM_XSTAR, B * n, -1, 1).reshape(B, n)
    rp, ci, _ = W.weighted_laplacian(n, ei, ej, w[0], 0.0)
    dpos = O.diag_positions(rp, ci)

    A = sla.CSR(T(rp), T(ci), batch=B, symmetric=True)
    E = sla.EdgeLaplacian(A, T(ei.astype(np.int32)), T(ej.astype(np.int32)))
    dpos_t = T(dpos.astype(np.int64))

    def residual(u, wt, kt, ft):
        return A.matvec(E.assemble(wt, shift), u) + kt * u ** 3 - ft

    def jacobian(u, wt, kt, ft):
        J = E.assemble_values(wt, shift).clone()
        J[:, dpos_t] += 3.0 * kt * u ** 2
        return J

    wt, kt, ft = T(w).requires_grad_(True), T(kappa).requires_grad_(True), T(f).requires_grad_(True)
    u = sla.newton_solve(A, residual, jacobian, torch.zeros(B, n, dtype=torch.float64, device=DEV),
                         wt, kt, ft, tol=1e-12, cg_rtol=1e-13)
    info = A.last_newton_info
    loss = 0.5 * ((u - T(uo)) ** 2).sum()
    loss.backward()

    vo = O.laplacian_assemble(rp, ci, ei, ej, w, shift)

    def res_np(U):
        return np.stack([O.spmv(rp, ci, vo[s], U[s]) for s in range(B)]) + kappa[0] * U ** 3 - f

    def jac_np(U):
        J = vo.copy()
        J[:, dpos] += 3.0 * kappa[0] * U ** 2
        return J

    u_o, info_o = O.newton(rp, ci, res_np, jac_np, np.zeros((B, n)), tol=1e-12, cg_rtol=1e-13)
    lam = O.newton_adjoint(rp, ci, jac_np(u_o), u_o - uo, cg_rtol=1e-13)
    G = O.grad_values(rp, ci, lam, u_o)                       # -lambda_i u_j
    dw_o, _ = O.laplacian_grad_values(rp, ci, ei, ej, G)      # -lambda^T dF/dw
    assert info.converged and info_o.converged
    assert info.steps == info_o.steps
    assert rel(H(u), u_o) < 1e-10
    assert rel(H(ft.grad), lam) < 1e-8                        # dF/df = -I
    assert abs(float(H(kt.grad)[0]) + float(np.sum(lam * u_o ** 3))) <= \
        1e-8 * abs(float(np.sum(lam * u_o ** 3)))
    assert rel(H(wt.grad), dw_o) < 1e-8
    # the backward ran one adjoint solve, whatever the number of Newton steps
    assert int(H(A.last_adjoint_info.status).max()) == 0


def test_newton_memory_does_not_depend_on_the_step_count():
    """The autograd graph of the solve is one node: peak memory of the backward
    is the same for 3 and for 12 Newton steps."""
    N = 64
    n = N * N
    rp, ci, v = W.poisson2d(N)
    A = sla.CSR(T(rp), T(ci), symmetric=True)
    vt = T(v)
    dpos_t = T(O.diag_positions(rp, ci).astype(np.int64))

    def residual(u, kt, ft):
        return A.matvec(vt, u) + kt * u ** 3 - ft

    def jacobian(u, kt, ft):
        J = vt.reshape(1, -1).clone()
        J[:, dpos_t] += 3.0 * kt * u ** 2
        return J

    peaks = []
    for tol in (1e-12, 1e-2, 1e-12):                 # the first run warms up
        kt = T(np.array([1.0])).requires_grad_(True)
        ft = T(50.0 * W.normal(92, W.STREAM_B, n)).requires_grad_(True)
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        u = sla.newton_solve(A, residual, jacobian, torch.zeros(n, dtype=torch.float64, device=DEV),
                             kt, ft, tol=tol)
        steps = A.last_newton_info.steps
        (0.5 * (u ** 2).sum()).backward()
        torch.cuda.synchronize()
        peaks.append((steps, torch.cuda.max_memory_allocated() - base))
        del u
    assert peaks[1][0] < peaks[2][0]
    assert peaks[1][1] == peaks[2][1]
