"""PyTorch surface of the library: a shared-pattern CSR matrix with
autograd-aware `solve` and `matvec`.

Mirrors the API of "torch-sla: Differentiable Sparse Linear Algebra with Adjoint
Solvers and Sparse Tensor Parallelism for PyTorch" (technical summary,
"Methodology" 1: `.solve`, `.matvec`, a SparseTensor holding one matrix or a
batch sharing one pattern; "Methodology" 2: the backward of a linear solve is
one adjoint solve A^T lambda = dL/dx, then dL/db = lambda and
dL/dA_ij = -lambda_i x_j on the pattern, so autograd stores O(1) nodes and
O(n + nnz) memory whatever the iteration count).

PyTorch provides device memory, streams and autograd bookkeeping; every step of
the computation runs in libsla.so's kernels (see _lib.py).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib as L


@dataclass
class SolveInfo:
    """Per-system outcome of a solve, kept on the device (no host sync)."""
    iters: torch.Tensor      # int32 [B]
    relres: torch.Tensor     # float64 [B]
    status: torch.Tensor     # int32 [B], see _lib.STATUS_NAMES


def _workspace(nbytes: int, device) -> torch.Tensor:
    # the caching allocator hands out blocks aligned to 512 bytes
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def _new_info(B: int, device) -> SolveInfo:
    return SolveInfo(torch.empty(B, dtype=torch.int32, device=device),
                     torch.empty(B, dtype=torch.float64, device=device),
                     torch.empty(B, dtype=torch.int32, device=device))


class CSR:
    """A CSR pattern on the GPU shared by ``batch`` value sets of one dtype.

    rowptr: int32 [n_rows + 1], colind: int32 [nnz] (device tensors, kept alive
    by this object).  Values and vectors are passed per call, batch-major:
    values [B, nnz] (or [nnz] when B == 1), vectors [B, n] (or [n]).
    ``symmetric=True`` asserts A^T == A for every value set, so the adjoint
    solve reuses the forward pattern and values unchanged.
    """

    def __init__(self, rowptr: torch.Tensor, colind: torch.Tensor, n_cols: int | None = None,
                 batch: int = 1, dtype: torch.dtype = torch.float64, symmetric: bool = False,
                 validate: bool = True, build_transpose: bool = False):
        if rowptr.device.type != "cuda" or colind.device.type != "cuda":
            raise ValueError("CSR needs CUDA tensors")
        self.rowptr = rowptr.to(torch.int32).contiguous()
        self.colind = colind.to(torch.int32).contiguous()
        self.n_rows = self.rowptr.numel() - 1
        self.n_cols = self.n_rows if n_cols is None else int(n_cols)
        self.nnz = self.colind.numel()
        self.batch = int(batch)
        self.dtype = dtype
        self.device = self.rowptr.device
        self.symmetric = bool(symmetric)
        flags = (L.SLA_FLAG_VALIDATE if validate else 0) | (L.SLA_FLAG_SYMMETRIC if symmetric else 0) \
            | (L.SLA_FLAG_BUILD_TRANSPOSE if build_transpose else 0)
        with torch.cuda.device(self.device):
            self.handle = L.sla_csr_create(self.n_rows, self.n_cols, self.nnz, self.rowptr, self.colind,
                                           self.batch, L.dtype_code(dtype), flags)
        self.last_info: SolveInfo | None = None
        self.last_adjoint_info: SolveInfo | None = None

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            try:
                torch.cuda.synchronize(self.device)
                L.sla_csr_destroy(h)
            except Exception:
                pass
            self.handle = None

    @property
    def props(self) -> L.sla_csr_props:
        return L.sla_csr_get_props(self.handle)

    # ------------------------------------------------------------ shapes
    def _values(self, values: torch.Tensor) -> torch.Tensor:
        v = values.reshape(self.batch, self.nnz)
        if v.dtype != self.dtype or v.device != self.device:
            raise TypeError(f"values must be {self.dtype} on {self.device}")
        return v.contiguous()

    def _vec(self, x: torch.Tensor, n: int) -> torch.Tensor:
        v = x.reshape(self.batch, n)
        if v.dtype != self.dtype or v.device != self.device:
            raise TypeError(f"vectors must be {self.dtype} on {self.device}")
        return v.contiguous()

    # -------------------------------------------------------- primitives
    def spmv(self, values, x, transpose: bool = False) -> torch.Tensor:
        """y = op(A) x without autograd (op = A or A^T)."""
        v = self._values(values)
        xin = self._vec(x, self.n_rows if transpose else self.n_cols)
        y = torch.empty(self.batch, self.n_cols if transpose else self.n_rows,
                        dtype=self.dtype, device=self.device)
        L.sla_spmv(self.handle, v, xin, y, int(transpose), 1.0, 0.0)
        return y

    def cg(self, values, b, *, adjoint=False, rtol=1e-10, atol=0.0, max_iter=0, fixed_iters=0,
           precond=True, x0=None, strategy=L.SLA_STRATEGY_AUTO, wait_timeout_ns=0):
        """Solve A x = b (or A^T x = b) without autograd; returns (x, SolveInfo)."""
        v = self._values(values)
        rhs = self._vec(b, self.n_rows)
        x = self._vec(x0, self.n_rows).clone() if x0 is not None else \
            torch.empty(self.batch, self.n_rows, dtype=self.dtype, device=self.device)
        info = _new_info(self.batch, self.device)
        opts = L.make_opts(rtol, atol, max_iter, fixed_iters, precond, x0 is not None,
                           wait_timeout_ns, strategy)
        op = L.SLA_OP_ADJOINT if adjoint else L.SLA_OP_CG
        ws = _workspace(L.sla_workspace_bytes(self.handle, op), self.device)
        fn = L.sla_cg_adjoint if adjoint else L.sla_cg_solve
        fn(self.handle, v, rhs, x, opts, L.make_info(info.iters, info.relres, info.status), ws)
        return x, info

    def grad_values(self, lam, x, out=None, accumulate=False) -> torch.Tensor:
        """dL/dvalues[t] = -lam[row t] * x[col t] on the pattern."""
        lm = self._vec(lam, self.n_rows)
        xv = self._vec(x, self.n_cols)
        g = out if out is not None else torch.empty(self.batch, self.nnz, dtype=self.dtype,
                                                    device=self.device)
        L.sla_grad_values(self.handle, lm, xv, g, int(accumulate))
        return g

    # ---------------------------------------------------- autograd calls
    def matvec(self, values, x) -> torch.Tensor:
        """y = A x, differentiable in values and x."""
        return _MatVec.apply(self, values, x)

    def solve(self, values, b, *, rtol=1e-10, atol=0.0, max_iter=0, fixed_iters=0, precond=True,
              strategy=L.SLA_STRATEGY_AUTO) -> torch.Tensor:
        """x = A^-1 b by Jacobi-PCG, differentiable in values and b through one
        adjoint solve with the same options."""
        opts = dict(rtol=rtol, atol=atol, max_iter=max_iter, fixed_iters=fixed_iters,
                    precond=precond, strategy=strategy)
        return _Solve.apply(self, values, b, opts)


class _MatVec(torch.autograd.Function):
    @staticmethod
    def forward(ctx, A: CSR, values, x):
        y = A.spmv(values, x)
        ctx.A = A
        ctx.save_for_backward(values, x)
        return y.reshape(x.shape[:-1] + (A.n_rows,))

    @staticmethod
    def backward(ctx, gy):
        A = ctx.A
        values, x = ctx.saved_tensors
        gv = gx = None
        gy = A._vec(gy, A.n_rows)
        if ctx.needs_input_grad[2]:
            gx = A.spmv(values, gy, transpose=True).reshape(x.shape)
        if ctx.needs_input_grad[1]:
            # dy_i/dA_ij = x_j, i.e. the value-gradient kernel with lambda = -gy
            gv = A.grad_values(-gy, x).reshape(values.shape)
        return None, gv, gx


class _Solve(torch.autograd.Function):
    @staticmethod
    def forward(ctx, A: CSR, values, b, opts):
        x, info = A.cg(values, b, **opts)
        A.last_info = info
        ctx.A, ctx.opts = A, opts
        ctx.save_for_backward(values, x)
        return x.reshape(b.shape)

    @staticmethod
    def backward(ctx, gx):
        A, opts = ctx.A, ctx.opts
        values, x = ctx.saved_tensors
        lam, info = A.cg(values, gx.contiguous(), adjoint=True, **opts)
        A.last_adjoint_info = info
        gv = A.grad_values(lam, x).reshape(values.shape) if ctx.needs_input_grad[1] else None
        gb = lam.reshape(gx.shape) if ctx.needs_input_grad[2] else None
        return None, gv, gb, None
