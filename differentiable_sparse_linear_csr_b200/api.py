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

import math
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
        self.n_info = self.batch                 # entries of a solve's SolveInfo
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
        info = _new_info(self.n_info, self.device)
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

    def matvec_grad_values(self, gy, x, out=None, accumulate=False) -> torch.Tensor:
        """dL/dvalues[t] = gy[row t] * x[col t] on the pattern (for y = A x)."""
        gv = self._vec(gy, self.n_rows)
        xv = self._vec(x, self.n_cols)
        g = out if out is not None else torch.empty(self.batch, self.nnz, dtype=self.dtype,
                                                    device=self.device)
        L.sla_matvec_grad_values(self.handle, gv, xv, g, int(accumulate))
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


class CSRList(CSR):
    """Independent square systems with their own patterns (torch-sla's
    SparseTensorList, technical summary, "Methodology" 1), held as one
    block-diagonal CSR: item s owns rows and columns [item_rows[s],
    item_rows[s+1]).  Values [nnz] and vectors [n_rows] are the items'
    concatenations; ``solve`` / ``cg`` solve every item on its own (SolveInfo
    per item), ``matvec`` and the gradients act item by item as they must for a
    block-diagonal matrix.  Build one with ``CSRList.from_items``.
    """

    def __init__(self, item_rows: torch.Tensor, rowptr: torch.Tensor, colind: torch.Tensor,
                 dtype: torch.dtype = torch.float64, symmetric: bool = False, validate: bool = True):
        if rowptr.device.type != "cuda" or colind.device.type != "cuda":
            raise ValueError("CSRList needs CUDA tensors")
        self.rowptr = rowptr.to(torch.int32).contiguous()
        self.colind = colind.to(torch.int32).contiguous()
        self.item_rows = item_rows.to(device=self.rowptr.device, dtype=torch.int32).contiguous()
        self.n_rows = self.n_cols = self.rowptr.numel() - 1
        self.nnz = self.colind.numel()
        self.batch = 1
        self.n_items = self.item_rows.numel() - 1
        self.dtype = dtype
        self.device = self.rowptr.device
        self.symmetric = bool(symmetric)
        flags = (L.SLA_FLAG_VALIDATE if validate else 0) | (L.SLA_FLAG_SYMMETRIC if symmetric else 0)
        with torch.cuda.device(self.device):
            self.handle = L.sla_csr_list_create(self.n_items, self.item_rows, self.n_rows, self.nnz,
                                                self.rowptr, self.colind, L.dtype_code(dtype), flags)
        self.n_info = self.n_items
        self.last_info = None
        self.last_adjoint_info = None

    @classmethod
    def from_items(cls, items, dtype=torch.float64, symmetric=False, validate=True, device=None):
        """items: sequence of (rowptr, colind) per item (local indices)."""
        rps, cis, rows, ents = [], [], [0], [0]
        for rp, ci in items:
            rp = torch.as_tensor(rp, dtype=torch.int64, device=device)
            ci = torch.as_tensor(ci, dtype=torch.int64, device=device)
            rps.append(rp[:-1] + ents[-1])
            cis.append(ci + rows[-1])
            rows.append(rows[-1] + rp.numel() - 1)
            ents.append(ents[-1] + ci.numel())
        rowptr = torch.cat(rps + [torch.tensor([ents[-1]], dtype=torch.int64, device=rps[0].device)])
        colind = torch.cat(cis)
        item_rows = torch.tensor(rows, dtype=torch.int64)
        dev = device or torch.device("cuda")
        return cls(item_rows.to(dev), rowptr.to(dev), colind.to(dev), dtype=dtype, symmetric=symmetric,
                   validate=validate)

    def split(self, t: torch.Tensor, per: str = "rows"):
        """Per-item views of a concatenated vector (per='rows') or of values
        (per='entries')."""
        bounds = self.item_rows.tolist() if per == "rows" else \
            self.rowptr[self.item_rows.long()].tolist()
        t = t.reshape(-1)
        return [t[a:b] for a, b in zip(bounds[:-1], bounds[1:])]


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
            gv = A.matvec_grad_values(gy, x).reshape(values.shape)   # dy_i/dA_ij = x_j
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


class EdgeLaplacian:
    """A = L_w + diag(shift) on the pattern of ``A``: the map from edge
    conductivities to matrix values of inverse coefficient learning ("torch-sla",
    technical summary, "Experimental results", end-to-end application).

    For undirected edges e = (ei[e], ej[e]) (int32 [E] device tensors, each pair
    once, both entries and every diagonal stored in the pattern):
    A_ij = A_ji = -w_e and A_ii = (i's edge weights, ascending neighbour index)
    + shift.  ``assemble`` and ``solve`` are differentiable in w, shift (and b);
    ``solve`` assembles, solves, and in its backward runs one adjoint solve and
    the fused edge-gradient kernel, never forming dL/dvalues.
    """

    def __init__(self, A: CSR, ei: torch.Tensor, ej: torch.Tensor):
        self.A = A
        self.ei = ei.to(device=A.device, dtype=torch.int32).contiguous()
        self.ej = ej.to(device=A.device, dtype=torch.int32).contiguous()
        self.n_edges = self.ei.numel()
        if self.ej.numel() != self.n_edges:
            raise ValueError("ei and ej must have the same length")
        with torch.cuda.device(A.device):
            self.plan = L.sla_edges_create(A.handle, self.n_edges, self.ei, self.ej)

    def __del__(self):
        p = getattr(self, "plan", None)
        if p:
            try:
                torch.cuda.synchronize(self.A.device)
                L.sla_edges_destroy(p)
            except Exception:
                pass
            self.plan = None

    def _w(self, w: torch.Tensor) -> torch.Tensor:
        A = self.A
        v = w.reshape(A.batch, self.n_edges)
        if v.dtype != A.dtype or v.device != A.device:
            raise TypeError(f"weights must be {A.dtype} on {A.device}")
        return v.contiguous()

    def _shift(self, shift):
        A = self.A
        if shift is None:
            return None
        if not torch.is_tensor(shift):
            return torch.full((A.batch,), float(shift), dtype=A.dtype, device=A.device)
        s = shift.reshape(-1)
        if s.numel() == 1 and A.batch > 1:
            s = s.expand(A.batch)
        if s.dtype != A.dtype or s.device != A.device:
            raise TypeError(f"shift must be {A.dtype} on {A.device}")
        return s.contiguous()

    # -------------------------------------------------------- primitives
    def assemble_values(self, w, shift=None) -> torch.Tensor:
        """values [B, nnz] of L_w + shift I, without autograd."""
        A = self.A
        vals = torch.empty(A.batch, A.nnz, dtype=A.dtype, device=A.device)
        L.sla_laplacian_assemble(self.plan, self._w(w), self._shift(shift), vals)
        return vals

    def _grads(self, fn, args, dw, dshift, accumulate, want_shift, shared_shift):
        A = self.A
        dw = dw if dw is not None else torch.empty(A.batch, self.n_edges, dtype=A.dtype, device=A.device)
        if dshift is None and want_shift:
            dshift = torch.empty(1 if shared_shift else A.batch, dtype=A.dtype, device=A.device)
        ws = _workspace(L.sla_edges_workspace_bytes(self.plan), A.device) if dshift is not None else None
        flags = (L.SLA_GRAD_ACCUMULATE if accumulate else 0) | \
            (L.SLA_GRAD_SHIFT_SHARED if shared_shift else 0)
        fn(self.plan, *args, dw, dshift, flags, ws)
        return dw, dshift

    def grad_from_values(self, G, dw=None, dshift=None, accumulate=False, want_shift=True,
                         shared_shift=False):
        """(dL/dw [B, E], dL/dshift [B]) from G = dL/dvalues by the chain rule;
        with shared_shift, dL/dshift [1] of one shift that serves every system."""
        return self._grads(L.sla_laplacian_grad_values, (self.A._values(G),), dw, dshift, accumulate,
                           want_shift, shared_shift)

    def grad(self, lam, x, dw=None, dshift=None, accumulate=False, want_shift=True, shared_shift=False):
        """The same for G = -lam x^T on the pattern, without forming G."""
        A = self.A
        return self._grads(L.sla_laplacian_grad, (A._vec(lam, A.n_rows), A._vec(x, A.n_rows)),
                           dw, dshift, accumulate, want_shift, shared_shift)

    # ---------------------------------------------------- autograd calls
    def assemble(self, w, shift=None) -> torch.Tensor:
        """values = L_w + shift I, differentiable in w and shift."""
        return _Assemble.apply(self, w, shift)

    def solve(self, w, b, shift=None, *, rtol=1e-10, atol=0.0, max_iter=0, fixed_iters=0,
              precond=True, strategy=L.SLA_STRATEGY_AUTO) -> torch.Tensor:
        """x = (L_w + shift I)^-1 b, differentiable in w, shift and b."""
        opts = dict(rtol=rtol, atol=atol, max_iter=max_iter, fixed_iters=fixed_iters,
                    precond=precond, strategy=strategy)
        return _EdgeSolve.apply(self, w, shift, b, opts)


class _Assemble(torch.autograd.Function):
    @staticmethod
    def forward(ctx, E: EdgeLaplacian, w, shift):
        ctx.E = E
        ctx.shift_shape = None if shift is None or not torch.is_tensor(shift) else shift.shape
        return E.assemble_values(w, shift).reshape(w.shape[:-1] + (E.A.nnz,))

    @staticmethod
    def backward(ctx, gv):
        E = ctx.E
        want_s = ctx.needs_input_grad[2]
        shared = want_s and math.prod(ctx.shift_shape) == 1 and E.A.batch > 1
        dw, ds = E.grad_from_values(gv.contiguous(), want_shift=want_s, shared_shift=shared)
        gw = dw.reshape(gv.shape[:-1] + (E.n_edges,)) if ctx.needs_input_grad[1] else None
        gs = ds.reshape(ctx.shift_shape) if want_s else None
        return None, gw, gs


class _EdgeSolve(torch.autograd.Function):
    @staticmethod
    def forward(ctx, E: EdgeLaplacian, w, shift, b, opts):
        A = E.A
        vals = E.assemble_values(w, shift)
        x, info = A.cg(vals, b, **opts)
        A.last_info = info
        ctx.E, ctx.opts = E, opts
        ctx.shift_shape = None if shift is None or not torch.is_tensor(shift) else shift.shape
        ctx.w_shape = w.shape
        ctx.save_for_backward(vals, x)
        return x.reshape(b.shape)

    @staticmethod
    def backward(ctx, gx):
        E, opts = ctx.E, ctx.opts
        A = E.A
        vals, x = ctx.saved_tensors
        lam, info = A.cg(vals, gx.contiguous(), adjoint=True, **opts)
        A.last_adjoint_info = info
        want_s = ctx.needs_input_grad[2]
        gw = gs = None
        if ctx.needs_input_grad[1] or want_s:
            shared = want_s and math.prod(ctx.shift_shape) == 1 and A.batch > 1
            dw, ds = E.grad(lam, x, want_shift=want_s, shared_shift=shared)
            gw = dw.reshape(ctx.w_shape) if ctx.needs_input_grad[1] else None
            if want_s:
                gs = ds.reshape(ctx.shift_shape)
        gb = lam.reshape(gx.shape) if ctx.needs_input_grad[3] else None
        return None, gw, gs, gb, None


@dataclass
class NewtonInfo:
    """Outcome of newton_solve (host values; each Newton step reads ||F||)."""
    steps: int
    residual_norms: list        # per step, the per-system ||F(u_k)||_2
    converged: bool
    linear: list                # per step, (iterations, statuses) of its linear solve


def newton_solve(A: CSR, residual, jacobian, u0, *theta, tol=1e-10, max_steps=50, cg_rtol=1e-12,
                 max_iter=0, precond=True, strategy=L.SLA_STRATEGY_AUTO) -> torch.Tensor:
    """u with F(u, theta) = 0 by Newton's method, differentiable in theta.

    Nonlinear systems of "torch-sla" (technical summary, "Methodology" 2): the
    Jacobian J = dF/du must be SPD with A's pattern (each Newton step is one
    Jacobi-PCG solve J delta = F, u <- u - delta); the backward pass is one
    adjoint solve J(u)^T lambda = dL/du and one vector-Jacobian product,
    dL/dtheta = -lambda^T dF/dtheta, whatever the number of Newton steps.

    theta are tensors; residual(u, *theta) -> F shaped like u (differentiable in
    theta, torch);
    jacobian(u, *theta) -> J's values [B, nnz] on A's pattern.  Stops when
    every system has ||F|| <= tol * max(1, ||F(u0)||).  A.last_newton_info
    holds the NewtonInfo of the last forward.
    """
    opts = dict(tol=tol, max_steps=max_steps, cg=dict(rtol=cg_rtol, max_iter=max_iter,
                                                      precond=precond, strategy=strategy))
    return _Newton.apply(A, residual, jacobian, opts, u0, *theta)


class _Newton(torch.autograd.Function):
    @staticmethod
    def forward(ctx, A: CSR, residual, jacobian, opts, u0, *theta):
        u = A._vec(u0, A.n_rows).clone()
        F = A._vec(residual(u, *theta), A.n_rows)
        # host copies only, so that nothing kept grows with the step count
        norms = [torch.linalg.vector_norm(F, dim=1).tolist()]
        bound = [opts["tol"] * max(1.0, v) for v in norms[0]]
        done = lambda nr: all(v <= t for v, t in zip(nr, bound))  # noqa: E731
        linear = []
        steps = 0
        while steps < opts["max_steps"] and not done(norms[-1]):
            Jv = A._values(jacobian(u, *theta))
            delta, info = A.cg(Jv, F, **opts["cg"])
            linear.append((info.iters.tolist(), info.status.tolist()))
            u.sub_(delta)
            del Jv, delta, info
            F = A._vec(residual(u, *theta), A.n_rows)
            norms.append(torch.linalg.vector_norm(F, dim=1).tolist())
            steps += 1
        A.last_newton_info = NewtonInfo(steps, norms, done(norms[-1]), linear)
        ctx.A, ctx.residual, ctx.jacobian, ctx.opts = A, residual, jacobian, opts
        ctx.u_shape = u0.shape
        ctx.save_for_backward(u, *theta)
        return u.reshape(u0.shape)

    @staticmethod
    def backward(ctx, gu):
        A, opts = ctx.A, ctx.opts
        u, *theta = ctx.saved_tensors
        needs = ctx.needs_input_grad[5:]
        if not any(needs):
            return (None,) * (5 + len(theta))
        with torch.no_grad():
            Jv = A._values(ctx.jacobian(u, *theta))
        lam, info = A.cg(Jv, A._vec(gu.contiguous(), A.n_rows), adjoint=True, **opts["cg"])
        A.last_adjoint_info = info
        with torch.enable_grad():
            th = [t.detach().requires_grad_(need) for t, need in zip(theta, needs)]
            F = ctx.residual(u.detach().reshape(ctx.u_shape), *th)
            wrt = [t for t, need in zip(th, needs) if need]
            got = torch.autograd.grad(F, wrt, grad_outputs=-lam.reshape(F.shape), allow_unused=True)
        it = iter(got)
        grads = [next(it) if need else None for need in needs]
        return (None, None, None, None, None, *grads)
