"""ctypes binding of libsla.so, the sm_100a library declared in include/sla.h.

Argument marshalling only: each function takes torch tensors (device memory),
passes their data pointers and the current CUDA stream to the C function of the
same name, and turns a non-OK status into SlaError.  Every computation runs in
the library's kernels; there is no fallback when the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

# SLA_LIBRARY_VARIANT=debug_bounds selects the bounds-checking build
# (libsla_debug_bounds.so); read once, when the library is first loaded.
_VARIANT = os.environ.get("SLA_LIBRARY_VARIANT", "")
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         f"libsla{'_' + _VARIANT if _VARIANT else ''}.so")

SLA_F64, SLA_F32 = 0, 1
SLA_OK, SLA_ERR_INVALID, SLA_ERR_CUDA, SLA_ERR_OOM, SLA_ERR_TIMEOUT, SLA_ERR_UNSUPPORTED = range(6)
SLA_CONVERGED, SLA_NOT_CONVERGED, SLA_BREAKDOWN, SLA_NONFINITE, SLA_FIXED_DONE, SLA_TIMED_OUT = range(6)
SLA_FLAG_VALIDATE, SLA_FLAG_SYMMETRIC, SLA_FLAG_BUILD_TRANSPOSE = 1, 2, 4
SLA_STRATEGY_AUTO, SLA_STRATEGY_GRID, SLA_STRATEGY_BLOCK, SLA_STRATEGY_CLUSTER = 0, 1, 2, 3
SLA_OP_SPMV, SLA_OP_CG, SLA_OP_ADJOINT, SLA_OP_GRAD = 0, 1, 2, 3
SLA_GRAD_ACCUMULATE, SLA_GRAD_SHIFT_SHARED = 1, 2

STATUS_NAMES = {0: "converged", 1: "not_converged", 2: "breakdown", 3: "nonfinite",
                4: "fixed_done", 5: "timed_out"}


class SlaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


class sla_cg_opts(ctypes.Structure):
    _fields_ = [("rtol", ctypes.c_double), ("atol", ctypes.c_double),
                ("max_iter", ctypes.c_int32), ("fixed_iters", ctypes.c_int32),
                ("precond", ctypes.c_int32), ("x0_given", ctypes.c_int32),
                ("wait_timeout_ns", ctypes.c_int64), ("strategy", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class sla_cg_info(ctypes.Structure):
    _fields_ = [("iters", ctypes.c_void_p), ("relres", ctypes.c_void_p),
                ("status", ctypes.c_void_p)]


class sla_csr_props(ctypes.Structure):
    _fields_ = [("n_rows", ctypes.c_int32), ("n_cols", ctypes.c_int32), ("nnz", ctypes.c_int64),
                ("batch", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("row_min", ctypes.c_int32), ("row_max", ctypes.c_int32),
                ("row_mean", ctypes.c_double), ("lanes", ctypes.c_int32),
                ("grid_blocks", ctypes.c_int32), ("block_fits", ctypes.c_int32),
                ("has_transpose", ctypes.c_int32), ("grid_onchip", ctypes.c_int32),
                ("grid_tile_rows", ctypes.c_int32), ("sliced", ctypes.c_int32),
                ("block_resident", ctypes.c_int32), ("cluster_fits", ctypes.c_int32),
                ("n_items", ctypes.c_int32), ("item_rows_max", ctypes.c_int32),
                ("item_smem_rows", ctypes.c_int32), ("sliced_col_bytes", ctypes.c_int32),
                ("interleaved", ctypes.c_int32)]


_P = ctypes.c_void_p
_I32, _I64, _U32, _F64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_double, ctypes.c_size_t

_SIGNATURES = {
    "sla_csr_create": ([_I32, _I32, _I64, _P, _P, _I32, _I32, _U32, _P, ctypes.POINTER(_P)], _I32),
    "sla_csr_destroy": ([_P], _I32),
    "sla_csr_get_props": ([_P, ctypes.POINTER(sla_csr_props)], _I32),
    "sla_csr_transpose_pattern": ([_P, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P), _P], _I32),
    "sla_workspace_bytes": ([_P, _I32], _SZ),
    "sla_spmv": ([_P, _P, _P, _P, _I32, _F64, _F64, _P], _I32),
    "sla_cg_solve": ([_P, _P, _P, _P, ctypes.POINTER(sla_cg_opts), sla_cg_info, _P, _SZ, _P], _I32),
    "sla_cg_adjoint": ([_P, _P, _P, _P, ctypes.POINTER(sla_cg_opts), sla_cg_info, _P, _SZ, _P], _I32),
    "sla_grad_values": ([_P, _P, _P, _P, _I32, _P], _I32),
    "sla_matvec_grad_values": ([_P, _P, _P, _P, _I32, _P], _I32),
    "sla_transpose_workspace_bytes": ([_I32, _I32, _I64], _SZ),
    "sla_csr_transpose": ([_I32, _I32, _I64, _P, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P], _I32),
    "sla_coo_workspace_bytes": ([_I32, _I32, _I64], _SZ),
    "sla_csr_from_coo": ([_I32, _I32, _I64, _P, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I32),
    "sla_csr_check": ([_I32, _I32, _I64, _P, _P, _I32, _P, _P], _I32),
    "sla_cg_solve_noalloc": ([_I32, _I64, _P, _P, _I32, _I32, _P, _P, _P, ctypes.POINTER(sla_cg_opts),
                              sla_cg_info, _P], _I32),
    "sla_csr_list_create": ([_I32, _P, _I32, _I64, _P, _P, _I32, _U32, _P, ctypes.POINTER(_P)], _I32),
    "sla_edges_create": ([_P, _I64, _P, _P, ctypes.POINTER(_I64), _P, ctypes.POINTER(_P)], _I32),
    "sla_edges_destroy": ([_P], _I32),
    "sla_laplacian_assemble": ([_P, _P, _P, _P, _P], _I32),
    "sla_edges_workspace_bytes": ([_P], _SZ),
    "sla_laplacian_grad_values": ([_P, _P, _P, _P, _I32, _P, _SZ, _P], _I32),
    "sla_laplacian_grad": ([_P, _P, _P, _P, _P, _I32, _P, _SZ, _P], _I32),
    "sla_debug_bounds_report": ([ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(_I32), ctypes.POINTER(_I64),
                                 _I32], _I32),
    "sla_last_error_string": ([], ctypes.c_char_p),
    "sla_version": ([], ctypes.c_char_p),
}

_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(
                f"{_LIB_PATH} is missing: build the CUDA library first "
                "(python -c 'import __graft_entry__ as g; g.build()' at the repository root)")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(fn: str, st: int) -> None:
    if st != SLA_OK:
        raise SlaError(fn, st, lib().sla_last_error_string().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    assert t.is_contiguous(), "tensors passed to the library must be contiguous"
    return t.data_ptr()


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.float64:
        return SLA_F64
    if dtype == torch.float32:
        return SLA_F32
    raise TypeError(f"unsupported value dtype {dtype} (float64 or float32)")


# --------------------------------------------------------------------------
# One function per C entry point, same names.
# --------------------------------------------------------------------------

def sla_debug_bounds_report(reset: bool = False) -> tuple[int, int, int]:
    """(violations, first code, first index) of the bounds-checking build."""
    v, c, i = ctypes.c_uint64(), _I32(), _I64()
    _check("sla_debug_bounds_report", lib().sla_debug_bounds_report(ctypes.byref(v), ctypes.byref(c),
                                                                    ctypes.byref(i), int(reset)))
    return int(v.value), int(c.value), int(i.value)


def sla_version() -> str:
    return lib().sla_version().decode()


def sla_last_error_string() -> str:
    return lib().sla_last_error_string().decode()


def sla_csr_create(n_rows, n_cols, nnz, rowptr, colind, batch, dtype, flags, stream=None) -> int:
    h = _P()
    _check("sla_csr_create", lib().sla_csr_create(n_rows, n_cols, nnz, _ptr(rowptr), _ptr(colind),
                                                  batch, dtype, flags, _stream(stream), ctypes.byref(h)))
    return h.value


def sla_csr_list_create(n_items, item_rows, n_rows, nnz, rowptr, colind, dtype, flags, stream=None) -> int:
    out = _P()
    _check("sla_csr_list_create", lib().sla_csr_list_create(
        n_items, _ptr(item_rows), n_rows, nnz, _ptr(rowptr), _ptr(colind), dtype, flags,
        _stream(stream), ctypes.byref(out)))
    return out.value


def sla_csr_destroy(h) -> None:
    _check("sla_csr_destroy", lib().sla_csr_destroy(h))


def sla_csr_get_props(h) -> sla_csr_props:
    p = sla_csr_props()
    _check("sla_csr_get_props", lib().sla_csr_get_props(h, ctypes.byref(p)))
    return p


def sla_csr_transpose_pattern(h, stream=None):
    rp, ci, pm = _P(), _P(), _P()
    _check("sla_csr_transpose_pattern", lib().sla_csr_transpose_pattern(
        h, ctypes.byref(rp), ctypes.byref(ci), ctypes.byref(pm), _stream(stream)))
    return rp.value, ci.value, pm.value


def sla_workspace_bytes(h, op) -> int:
    return int(lib().sla_workspace_bytes(h, op))


def sla_spmv(h, vals, x, y, transpose=0, alpha=1.0, beta=0.0, stream=None) -> None:
    _check("sla_spmv", lib().sla_spmv(h, _ptr(vals), _ptr(x), _ptr(y), int(transpose),
                                      float(alpha), float(beta), _stream(stream)))


def make_opts(rtol=1e-10, atol=0.0, max_iter=0, fixed_iters=0, precond=True, x0_given=False,
              wait_timeout_ns=0, strategy=SLA_STRATEGY_AUTO) -> sla_cg_opts:
    return sla_cg_opts(float(rtol), float(atol), int(max_iter), int(fixed_iters), int(bool(precond)),
                       int(bool(x0_given)), int(wait_timeout_ns), int(strategy), 0)


def make_info(iters=None, relres=None, status=None) -> sla_cg_info:
    return sla_cg_info(_ptr(iters), _ptr(relres), _ptr(status))


def sla_cg_solve(h, vals, b, x, opts, info, ws, stream=None) -> None:
    _check("sla_cg_solve", lib().sla_cg_solve(h, _ptr(vals), _ptr(b), _ptr(x), ctypes.byref(opts),
                                              info, _ptr(ws), ws.numel() * ws.element_size(),
                                              _stream(stream)))


def sla_cg_adjoint(h, vals, g, lam, opts, info, ws, stream=None) -> None:
    _check("sla_cg_adjoint", lib().sla_cg_adjoint(h, _ptr(vals), _ptr(g), _ptr(lam), ctypes.byref(opts),
                                                  info, _ptr(ws), ws.numel() * ws.element_size(),
                                                  _stream(stream)))


def sla_grad_values(h, lam, x, grad, accumulate=0, stream=None) -> None:
    _check("sla_grad_values", lib().sla_grad_values(h, _ptr(lam), _ptr(x), _ptr(grad), int(accumulate),
                                                    _stream(stream)))


def sla_matvec_grad_values(h, gy, x, grad, accumulate=0, stream=None) -> None:
    _check("sla_matvec_grad_values", lib().sla_matvec_grad_values(h, _ptr(gy), _ptr(x), _ptr(grad),
                                                                  int(accumulate), _stream(stream)))


def sla_transpose_workspace_bytes(n_rows, n_cols, nnz) -> int:
    return int(lib().sla_transpose_workspace_bytes(n_rows, n_cols, nnz))


def sla_csr_transpose(n_rows, n_cols, nnz, rowptr, colind, batch, dtype, vals, rowptrT, colindT,
                      valsT, perm, ws, stream=None) -> None:
    _check("sla_csr_transpose", lib().sla_csr_transpose(
        n_rows, n_cols, nnz, _ptr(rowptr), _ptr(colind), batch, dtype, _ptr(vals), _ptr(rowptrT),
        _ptr(colindT), _ptr(valsT), _ptr(perm), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def sla_coo_workspace_bytes(n_rows, n_cols, nnz_in) -> int:
    return int(lib().sla_coo_workspace_bytes(n_rows, n_cols, nnz_in))


def sla_csr_from_coo(n_rows, n_cols, nnz_in, row, col, batch, dtype, val, rowptr, colind, val_out,
                     slot, nnz_out, ws, stream=None) -> None:
    _check("sla_csr_from_coo", lib().sla_csr_from_coo(
        n_rows, n_cols, nnz_in, _ptr(row), _ptr(col), batch, dtype, _ptr(val), _ptr(rowptr),
        _ptr(colind), _ptr(val_out), _ptr(slot), _ptr(nnz_out), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def sla_csr_check(n_rows, n_cols, nnz, rowptr, colind, need_diag, result, stream=None) -> None:
    _check("sla_csr_check", lib().sla_csr_check(n_rows, n_cols, nnz, _ptr(rowptr), _ptr(colind),
                                                int(need_diag), _ptr(result), _stream(stream)))


def sla_cg_solve_noalloc(n, nnz, rowptr, colind, batch, dtype, vals, b, x, opts, info, stream=None) -> None:
    """Allocation-free solve: scratch in the library's static device array (no workspace)."""
    _check("sla_cg_solve_noalloc", lib().sla_cg_solve_noalloc(
        n, nnz, _ptr(rowptr), _ptr(colind), batch, dtype, _ptr(vals), _ptr(b), _ptr(x),
        ctypes.byref(opts), info, _stream(stream)))


class EdgeCheckError(SlaError):
    """Invalid edge list: ``code`` and ``index`` as documented in include/sla.h."""
    def __init__(self, fn: str, status: int, msg: str, check: int):
        super().__init__(fn, status, msg)
        self.code = check >> 40
        self.index = check & ((1 << 40) - 1)


def sla_edges_create(h, n_edges, ei, ej, stream=None) -> int:
    out = _P()
    check = _I64(0)
    st = lib().sla_edges_create(h, n_edges, _ptr(ei), _ptr(ej), ctypes.byref(check), _stream(stream),
                                ctypes.byref(out))
    if st != SLA_OK:
        msg = lib().sla_last_error_string().decode()
        if check.value:
            raise EdgeCheckError("sla_edges_create", st, msg, check.value)
        raise SlaError("sla_edges_create", st, msg)
    return out.value


def sla_edges_destroy(e) -> None:
    _check("sla_edges_destroy", lib().sla_edges_destroy(e))


def sla_laplacian_assemble(e, w, shift, vals, stream=None) -> None:
    _check("sla_laplacian_assemble", lib().sla_laplacian_assemble(e, _ptr(w), _ptr(shift), _ptr(vals),
                                                                  _stream(stream)))


def sla_edges_workspace_bytes(e) -> int:
    return int(lib().sla_edges_workspace_bytes(e))


def sla_laplacian_grad_values(e, G, dw, dshift, flags, ws, stream=None) -> None:
    _check("sla_laplacian_grad_values", lib().sla_laplacian_grad_values(
        e, _ptr(G), _ptr(dw), _ptr(dshift), int(flags), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def sla_laplacian_grad(e, lam, x, dw, dshift, flags, ws, stream=None) -> None:
    _check("sla_laplacian_grad", lib().sla_laplacian_grad(
        e, _ptr(lam), _ptr(x), _ptr(dw), _ptr(dshift), int(flags), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))
