"""ctypes wrapper of the plain-C CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY.  The oracle is the slow, obviously correct definition
of the sparse SPD solve of "torch-sla: Differentiable Sparse Linear Algebra with
Adjoint Solvers and Sparse Tensor Parallelism for PyTorch" (technical summary,
"Methodology" 1: the `.solve` / `.matvec` API with an iterative Jacobi-CG
backend; "Methodology" 2: the linear adjoint, A^T lambda = dL/dx and
dL/dA_ij = -lambda_i x_j on the pattern).  Only the tests, the package smoke
check and the benchmark's CPU-baseline leg use it; it imports nothing from the
CUDA package and the CUDA package never imports it.

Batched inputs ([B][...]) are handled here by a plain loop over systems.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BODY = os.path.join(_HERE, "oracle_body.h")
_LIB = os.path.join(_HERE, "liboracle.so")
_LIB_OMP = os.path.join(_HERE, "liboracle_omp.so")

CONVERGED, NOT_CONVERGED, BREAKDOWN, NONFINITE, FIXED_DONE = 0, 1, 2, 3, 4


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, contraction off).

    openmp=True builds liboracle_omp.so from the same source with -fopenmp, for
    the benchmark's all-cores CPU baseline only: rows and vector entries are
    split over threads (same arithmetic) and dot products are summed per thread
    before they are combined (another order of the same additions)."""
    lib = _LIB_OMP if openmp else _LIB
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_BODY))
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < newest:
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC",
                               *(["-fopenmp"] if openmp else []), "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, lib)
    return lib


class _Opts(ctypes.Structure):
    _fields_ = [("rtol", ctypes.c_double), ("atol", ctypes.c_double),
                ("max_iter", ctypes.c_int32), ("fixed_iters", ctypes.c_int32),
                ("precond", ctypes.c_int32), ("x0_given", ctypes.c_int32),
                ("reverse_order", ctypes.c_int32)]


class _Result(ctypes.Structure):
    _fields_ = [("iters", ctypes.c_int32), ("status", ctypes.c_int32),
                ("relres", ctypes.c_double)]


_lib = None


def _L():
    """The oracle library: the single-threaded build, or the OpenMP build when
    the environment variable SLA_ORACLE_OPENMP=1 is set before first use."""
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build(openmp=os.environ.get("SLA_ORACLE_OPENMP") == "1"))
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        for sfx in ("f64", "f32"):
            getattr(_lib, f"orc_spmv_{sfx}").argtypes = [i32, P, P, P, P, P, i32]
            getattr(_lib, f"orc_pcg_{sfx}").argtypes = [i32, P, P, P, P, P, P, P]
            getattr(_lib, f"orc_pcg_{sfx}").restype = i32
            getattr(_lib, f"orc_cg_adjoint_{sfx}").argtypes = [i32, P, P, P, P, P, P, P]
            getattr(_lib, f"orc_cg_adjoint_{sfx}").restype = i32
            getattr(_lib, f"orc_grad_values_{sfx}").argtypes = [i32, P, P, P, P, P, i32]
            getattr(_lib, f"orc_coo_to_csr_{sfx}").argtypes = [i32, i32, i64, P, P, P, P, P, P, P]
            getattr(_lib, f"orc_coo_to_csr_{sfx}").restype = i64
            ft = ctypes.c_double if sfx == "f64" else ctypes.c_float
            getattr(_lib, f"orc_laplacian_assemble_{sfx}").argtypes = [i32, P, P, P, P, ft, P]
            getattr(_lib, f"orc_laplacian_grad_values_{sfx}").argtypes = [i32, P, P, i64, P, P, P, P,
                                                                          P, P, P, i32]
        _lib.orc_edge_slots.argtypes = [i32, P, P, i64, P, P, P, P, P, P]
        _lib.orc_edge_slots.restype = i32
        _lib.orc_transpose_pattern.argtypes = [i32, i32, P, P, P, P, P]
        _lib.orc_coo_order.argtypes = [i32, i32, i64, P, P, P]
        _lib.orc_csr_check.argtypes = [i32, i32, i64, P, P, i32, P]
        _lib.orc_csr_check.restype = i32
        _lib.orc_diag_positions.argtypes = [i32, P, P, P]
        _lib.orc_dense_lu_solve.argtypes = [i32, P, P]
        _lib.orc_dense_lu_solve.restype = i32
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _sfx(dtype) -> str:
    dt = np.dtype(dtype)
    if dt == np.float64:
        return "f64"
    if dt == np.float32:
        return "f32"
    raise TypeError(f"oracle supports float64/float32, not {dt}")


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _batch(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return (a[None, :], True) if a.ndim == 1 else (a, False)


def spmv(rowptr, colind, vals, x, reverse: bool = False) -> np.ndarray:
    """y = A x per system; vals [B][nnz] (or [nnz]), x [B][n_cols] (or [n_cols])."""
    rowptr, colind = _i32(rowptr), _i32(colind)
    dt = np.asarray(vals).dtype
    V, single = _batch(vals, dt)
    X, _ = _batch(x, dt)
    n = rowptr.shape[0] - 1
    Y = np.empty((V.shape[0], n), dtype=dt)
    f = getattr(_L(), f"orc_spmv_{_sfx(dt)}")
    for b in range(V.shape[0]):
        xb = np.ascontiguousarray(X[b if X.shape[0] > 1 else 0])
        yb = np.empty(n, dtype=dt)
        f(n, _p(rowptr), _p(colind), _p(np.ascontiguousarray(V[b])), _p(xb), _p(yb), int(reverse))
        Y[b] = yb
    return Y[0] if single else Y


@dataclass
class SolveInfo:
    iters: np.ndarray
    status: np.ndarray
    relres: np.ndarray


def _solve(fname, rowptr, colind, vals, rhs, *, rtol=1e-10, atol=0.0, max_iter=None,
           fixed_iters=0, precond=True, x0=None, reverse=False):
    rowptr, colind = _i32(rowptr), _i32(colind)
    dt = np.asarray(vals).dtype
    V, single = _batch(vals, dt)
    Bv, _ = _batch(rhs, dt)
    n = rowptr.shape[0] - 1
    nsys = max(V.shape[0], Bv.shape[0])
    if max_iter is None:
        max_iter = min(10 * n, 100_000)
    X = np.zeros((nsys, n), dtype=dt)
    if x0 is not None:
        X0, _ = _batch(x0, dt)
        X[:] = X0
    iters = np.zeros(nsys, np.int32)
    status = np.zeros(nsys, np.int32)
    relres = np.zeros(nsys, np.float64)
    f = getattr(_L(), f"{fname}_{_sfx(dt)}")
    o = _Opts(rtol, atol, max_iter, fixed_iters, int(precond), int(x0 is not None), int(reverse))
    for s in range(nsys):
        vb = np.ascontiguousarray(V[s if V.shape[0] > 1 else 0])
        bb = np.ascontiguousarray(Bv[s if Bv.shape[0] > 1 else 0])
        xb = np.ascontiguousarray(X[s])
        r = _Result()
        rc = f(n, _p(rowptr), _p(colind), _p(vb), _p(bb), _p(xb), ctypes.byref(o), ctypes.byref(r))
        if rc != 0:
            raise MemoryError("oracle allocation failed")
        X[s] = xb
        iters[s], status[s], relres[s] = r.iters, r.status, r.relres
    info = SolveInfo(iters, status, relres)
    return (X[0] if single and Bv.ndim == 2 and nsys == 1 and np.asarray(rhs).ndim == 1 else X), info


def pcg(rowptr, colind, vals, b, **kw):
    """Jacobi-PCG solve of A x = b; returns (x, SolveInfo).  See oracle_body.h."""
    return _solve("orc_pcg", rowptr, colind, vals, b, **kw)


def cg_adjoint(rowptr, colind, vals, g, **kw):
    """Adjoint solve A^T lambda = g on an explicitly transposed pattern."""
    return _solve("orc_cg_adjoint", rowptr, colind, vals, g, **kw)


def grad_values(rowptr, colind, lam, x, grad=None) -> np.ndarray:
    """dL/dvals[t] = -lambda[row t] * x[col t]; added to ``grad`` when given."""
    rowptr, colind = _i32(rowptr), _i32(colind)
    dt = np.asarray(lam).dtype
    Lm, single = _batch(lam, dt)
    X, _ = _batch(x, dt)
    nnz = colind.shape[0]
    G = np.zeros((Lm.shape[0], nnz), dtype=dt) if grad is None else _batch(grad, dt)[0].copy()
    f = getattr(_L(), f"orc_grad_values_{_sfx(dt)}")
    for s in range(Lm.shape[0]):
        gb = np.ascontiguousarray(G[s])
        f(rowptr.shape[0] - 1, _p(rowptr), _p(colind), _p(np.ascontiguousarray(Lm[s])),
          _p(np.ascontiguousarray(X[s])), _p(gb), int(grad is not None))
        G[s] = gb
    return G[0] if single else G


def transpose(rowptr, colind, vals, n_cols: int | None = None):
    """A^T in CSR by stable counting sort; returns (rowptrT, colindT, valsT, perm)."""
    rowptr, colind = _i32(rowptr), _i32(colind)
    n_rows = rowptr.shape[0] - 1
    n_cols = n_rows if n_cols is None else n_cols
    nnz = colind.shape[0]
    rpT = np.zeros(n_cols + 1, np.int32)
    ciT = np.zeros(nnz, np.int32)
    perm = np.zeros(nnz, np.int64)
    _L().orc_transpose_pattern(n_rows, n_cols, _p(rowptr), _p(colind), _p(rpT), _p(ciT), _p(perm))
    v = np.asarray(vals)
    return rpT, ciT, np.ascontiguousarray(v[..., perm]), perm


def coo_to_csr(n_rows: int, n_cols: int, row, col, val):
    """COO -> CSR, duplicates summed in input order; returns (rowptr, colind, vals, slot)."""
    row, col = _i32(row), _i32(col)
    dt = np.asarray(val).dtype
    V, single = _batch(val, dt)
    nnz_in = row.shape[0]
    f = getattr(_L(), f"orc_coo_to_csr_{_sfx(dt)}")
    outs = []
    for s in range(V.shape[0]):
        rp = np.zeros(n_rows + 1, np.int32)
        ci = np.zeros(max(nnz_in, 1), np.int32)
        vo = np.zeros(max(nnz_in, 1), dt)
        slot = np.zeros(max(nnz_in, 1), np.int64)
        m = f(n_rows, n_cols, nnz_in, _p(row), _p(col), _p(np.ascontiguousarray(V[s])),
              _p(rp), _p(ci), _p(vo), _p(slot))
        outs.append((rp, ci[:m].copy(), vo[:m].copy(), slot[:nnz_in].copy()))
    rp, ci, _, slot = outs[0]
    vals = np.stack([o[2] for o in outs])
    return rp, ci, (vals[0] if single else vals), slot


def csr_check(n_rows, n_cols, rowptr, colind, need_diag=False):
    """Returns (code, where) as documented in oracle.c; code 0 means valid."""
    rowptr, colind = _i32(rowptr), _i32(colind)
    where = np.zeros(1, np.int64)
    code = _L().orc_csr_check(n_rows, n_cols, colind.shape[0], _p(rowptr), _p(colind),
                              int(need_diag), _p(where))
    return int(code), int(where[0])


def diag_positions(rowptr, colind) -> np.ndarray:
    rowptr, colind = _i32(rowptr), _i32(colind)
    d = np.zeros(rowptr.shape[0] - 1, np.int32)
    _L().orc_diag_positions(rowptr.shape[0] - 1, _p(rowptr), _p(colind), _p(d))
    return d


@dataclass
class EdgeSlots:
    code: int               # 0, or the failure code documented in oracle.c
    where: int              # offending edge (or row, code 5); -1 when valid
    slot_ij: np.ndarray     # int64 [E]: position of entry (i, j)
    slot_ji: np.ndarray     # int64 [E]: position of entry (j, i)
    owner: np.ndarray       # int64 [nnz]: edge carried by each entry, -1 for none


def edge_slots(rowptr, colind, ei, ej) -> EdgeSlots:
    """Pattern positions of undirected edges (see orc_edge_slots)."""
    rowptr, colind, ei, ej = _i32(rowptr), _i32(colind), _i32(ei), _i32(ej)
    E = ei.shape[0]
    sij, sji = np.zeros(max(E, 1), np.int64), np.zeros(max(E, 1), np.int64)
    owner = np.zeros(max(colind.shape[0], 1), np.int64)
    where = np.zeros(1, np.int64)
    code = _L().orc_edge_slots(rowptr.shape[0] - 1, _p(rowptr), _p(colind), E, _p(ei), _p(ej),
                               _p(sij), _p(sji), _p(owner), _p(where))
    return EdgeSlots(int(code), int(where[0]), sij[:E], sji[:E], owner[:colind.shape[0]])


def _shifts(shift, B, dt):
    s = np.zeros(B, dt) if shift is None else np.broadcast_to(np.asarray(shift, dt), (B,))
    return [dt.type(v) for v in s]


def laplacian_assemble(rowptr, colind, ei, ej, w, shift=None) -> np.ndarray:
    """Values of L_w + shift*I on the pattern; w [E] or [B][E], shift scalar or [B]."""
    rowptr, colind = _i32(rowptr), _i32(colind)
    es = edge_slots(rowptr, colind, ei, ej)
    if es.code != 0:
        raise ValueError(f"invalid edges: code {es.code} at {es.where}")
    dt = np.asarray(w).dtype
    W, single = _batch(w, dt)
    f = getattr(_L(), f"orc_laplacian_assemble_{_sfx(dt)}")
    V = np.zeros((W.shape[0], colind.shape[0]), dt)
    for s, sh in enumerate(_shifts(shift, W.shape[0], np.dtype(dt))):
        vb = np.zeros(max(colind.shape[0], 1), dt)
        f(rowptr.shape[0] - 1, _p(rowptr), _p(colind), _p(es.owner if es.owner.size else
                                                        np.zeros(1, np.int64)),
          _p(np.ascontiguousarray(W[s])), sh, _p(vb))
        V[s] = vb[:colind.shape[0]]
    return V[0] if single else V


def laplacian_grad_values(rowptr, colind, ei, ej, G, dw=None, dshift=None):
    """Chain rule through laplacian_assemble: returns (dL/dw [.., E], dL/dshift [..]).
    With dw / dshift given, the results are added to copies of them."""
    rowptr, colind, ei, ej = _i32(rowptr), _i32(colind), _i32(ei), _i32(ej)
    es = edge_slots(rowptr, colind, ei, ej)
    if es.code != 0:
        raise ValueError(f"invalid edges: code {es.code} at {es.where}")
    dt = np.asarray(G).dtype
    Gb, single = _batch(G, dt)
    B, E = Gb.shape[0], ei.shape[0]
    acc = dw is not None
    DW = _batch(dw, dt)[0].copy() if acc else np.zeros((B, E), dt)
    DS = np.broadcast_to(np.asarray(dshift, dt), (B,)).copy() if dshift is not None else np.zeros(B, dt)
    f = getattr(_L(), f"orc_laplacian_grad_values_{_sfx(dt)}")
    for s in range(B):
        dws = np.ascontiguousarray(DW[s]) if E else np.zeros(1, dt)
        dss = np.array([DS[s]], dt)
        f(rowptr.shape[0] - 1, _p(rowptr), _p(colind), E, _p(ei if E else np.zeros(1, np.int32)),
          _p(ej if E else np.zeros(1, np.int32)), _p(es.slot_ij if E else np.zeros(1, np.int64)),
          _p(es.slot_ji if E else np.zeros(1, np.int64)), _p(np.ascontiguousarray(Gb[s])), _p(dws),
          _p(dss), int(acc or dshift is not None))
        DW[s] = dws[:E]
        DS[s] = dss[0]
    return (DW[0], DS[0]) if single else (DW, DS)


def dense_lu_solve(a, b) -> np.ndarray:
    """Dense Gaussian elimination with partial pivoting (tiny pins only)."""
    a = np.array(a, dtype=np.float64, order="C")
    x = np.array(b, dtype=np.float64)
    if _L().orc_dense_lu_solve(a.shape[0], _p(a), _p(x)) != 0:
        raise np.linalg.LinAlgError("singular matrix")
    return x


@dataclass
class NewtonInfo:
    steps: int                  # Newton steps taken
    residual_norms: list        # ||F(u_k)||_2 of system 0..B-1 at every step, k = 0..steps
    converged: bool


def newton(rowptr, colind, residual, jacobian, u0, *, tol=1e-10, max_steps=50, cg_rtol=1e-13):
    """Newton's method for F(u) = 0 with a sparse SPD Jacobian on the pattern
    (nonlinear systems of torch-sla, technical summary, "Methodology" 2): the
    plain iteration u <- u - J(u)^-1 F(u), each linear solve by the oracle's
    PCG.  residual(u) -> F [B][n] and jacobian(u) -> values [B][nnz] are numpy
    callables; stops when every system has ||F(u)|| <= tol * max(1, ||F(u0)||)."""
    u = np.array(u0, dtype=np.float64, copy=True)
    single = u.ndim == 1
    U = u[None, :] if single else u
    F = np.atleast_2d(residual(U))
    norms = [np.linalg.norm(F, axis=1)]
    bound = tol * np.maximum(1.0, norms[0])
    steps = 0
    while not np.all(norms[-1] <= bound) and steps < max_steps:
        Jv = np.atleast_2d(jacobian(U))
        delta, _ = pcg(rowptr, colind, Jv, F, rtol=cg_rtol)
        U = U - np.atleast_2d(delta)
        F = np.atleast_2d(residual(U))
        norms.append(np.linalg.norm(F, axis=1))
        steps += 1
    info = NewtonInfo(steps, [n.tolist() for n in norms], bool(np.all(norms[-1] <= bound)))
    return (U[0] if single else U), info


def newton_adjoint(rowptr, colind, jac_values, gu, *, cg_rtol=1e-13):
    """The adjoint of F(u, theta) = 0 at its solution: J^T lambda = dL/du (one
    oracle adjoint solve); then dL/dtheta = -lambda^T dF/dtheta is the caller's
    vector-Jacobian product with -lambda."""
    lam, _ = cg_adjoint(rowptr, colind, jac_values, gu, rtol=cg_rtol)
    return lam


def _items(item_rows, rowptr, colind):
    """Each item's own CSR (local row and column numbers) and its row / entry ranges."""
    item_rows, rowptr, colind = np.asarray(item_rows), _i32(rowptr), _i32(colind)
    for s in range(item_rows.shape[0] - 1):
        o, e = int(item_rows[s]), int(item_rows[s + 1])
        t0, t1 = int(rowptr[o]), int(rowptr[e])
        yield o, e, t0, t1, (rowptr[o:e + 1] - t0).astype(np.int32), (colind[t0:t1] - o).astype(np.int32)


def pcg_list(item_rows, rowptr, colind, vals, b, *, adjoint=False, **kw):
    """Independent Jacobi-PCG solves of the items of a block-diagonal CSR
    (torch-sla's SparseTensorList, technical summary, "Methodology" 1): item s
    owns rows and columns [item_rows[s], item_rows[s+1]).  Returns the
    concatenated solution and a SolveInfo with one entry per item."""
    vals, b = np.asarray(vals), np.asarray(b)
    x = np.zeros_like(b)
    iters, status, relres = [], [], []
    x0 = kw.pop("x0", None)
    for o, e, t0, t1, rp, ci in _items(item_rows, rowptr, colind):
        if x0 is not None:
            kw["x0"] = np.asarray(x0)[o:e]
        fn = cg_adjoint if adjoint else pcg
        xs, info = fn(rp, ci, vals[t0:t1], b[o:e], **kw)
        x[o:e] = xs
        iters.append(int(np.atleast_1d(info.iters)[0]))
        status.append(int(np.atleast_1d(info.status)[0]))
        relres.append(float(np.atleast_1d(info.relres)[0]))
    return x, SolveInfo(np.array(iters), np.array(status), np.array(relres))
