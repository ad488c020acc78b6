"""B200-native differentiable sparse SPD solves on CSR matrices.

Jacobi-preconditioned conjugate gradient with the implicit-function-theorem
adjoint and the sparse value gradient, as hand-written sm_100a CUDA kernels
behind a C ABI (include/sla.h), with a PyTorch autograd surface (api.CSR), and
the edge-weighted Laplacian with its chain rule to edge weights
(api.EdgeLaplacian), and Newton solves of F(u, theta) = 0 with the nonlinear
adjoint (api.newton_solve).
The CUDA library is loaded on first use and is required: there is no CPU path.
"""
from .api import CSR, CSRList, EdgeLaplacian, NewtonInfo, SolveInfo, newton_solve  # noqa: F401
from . import _lib  # noqa: F401

__all__ = ["CSR", "CSRList", "EdgeLaplacian", "NewtonInfo", "SolveInfo", "newton_solve"]
