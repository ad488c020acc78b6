"""The C-ABI library loads and exports every declared entry point; host-side
argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from differentiable_sparse_linear_csr_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "sla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sla_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = _declared_functions()
    for required in ("sla_csr_create", "sla_spmv", "sla_cg_solve", "sla_cg_adjoint",
                     "sla_grad_values", "sla_csr_transpose", "sla_csr_from_coo"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = L.lib()
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared_functions()) <= set(L._SIGNATURES), "binding lacks a declared call"


def test_version_and_error_string():
    assert "sm_100a" in L.sla_version()
    assert isinstance(L.sla_last_error_string(), str)


def test_host_side_argument_errors_need_no_gpu():
    lib = L.lib()
    h = ctypes.c_void_p()
    st = lib.sla_csr_create(4, 4, 8, None, None, 1, 0, 0, None, ctypes.byref(h))
    assert st == L.SLA_ERR_INVALID and h.value is None
    assert "rowptr" in L.sla_last_error_string()
    st = lib.sla_csr_create(-1, 4, 0, ctypes.c_void_p(256), None, 1, 0, 0, None, ctypes.byref(h))
    assert st == L.SLA_ERR_INVALID
    st = lib.sla_csr_create(4, 4, 0, ctypes.c_void_p(256), None, 0, 0, 0, None, ctypes.byref(h))
    assert st == L.SLA_ERR_INVALID and "batch" in L.sla_last_error_string()
    st = lib.sla_csr_create(4, 4, 0, ctypes.c_void_p(256), None, 1, 7, 0, None, ctypes.byref(h))
    assert st == L.SLA_ERR_INVALID and "dtype" in L.sla_last_error_string()
    st = lib.sla_csr_create(4, 5, 0, ctypes.c_void_p(256), None, 1, 0, L.SLA_FLAG_SYMMETRIC, None,
                            ctypes.byref(h))
    assert st == L.SLA_ERR_INVALID and "square" in L.sla_last_error_string()
    assert lib.sla_spmv(None, None, None, None, 0, 1.0, 0.0, None) == L.SLA_ERR_INVALID
    assert lib.sla_grad_values(None, None, None, None, 0, None) == L.SLA_ERR_INVALID
    assert lib.sla_matvec_grad_values(None, None, None, None, 0, None) == L.SLA_ERR_INVALID
    assert "sla_matvec_grad_values" in L.sla_last_error_string()
    opts = L.make_opts()
    info = L.make_info()
    assert lib.sla_cg_solve(None, None, None, None, ctypes.byref(opts), info, None, 0, None) == L.SLA_ERR_INVALID
    assert lib.sla_cg_adjoint(None, None, None, None, ctypes.byref(opts), info, None, 0, None) == L.SLA_ERR_INVALID
    assert lib.sla_workspace_bytes(None, L.SLA_OP_CG) == 0
    assert lib.sla_csr_destroy(None) == L.SLA_OK
    e = ctypes.c_void_p()
    check = ctypes.c_int64(7)
    assert lib.sla_edges_create(None, 0, None, None, ctypes.byref(check), None,
                                ctypes.byref(e)) == L.SLA_ERR_INVALID
    assert e.value is None and check.value == 0 and "handle" in L.sla_last_error_string()
    assert lib.sla_laplacian_assemble(None, None, None, None, None) == L.SLA_ERR_INVALID
    assert lib.sla_laplacian_grad_values(None, None, None, None, 0, None, 0, None) == L.SLA_ERR_INVALID
    assert lib.sla_laplacian_grad(None, None, None, None, None, 0, None, 0, None) == L.SLA_ERR_INVALID
    for fn in (lib.sla_laplacian_grad_values, lib.sla_laplacian_grad):
        args = [None] * (8 if fn is lib.sla_laplacian_grad_values else 9)
        fl = 4 if fn is lib.sla_laplacian_grad_values else 5
        args[fl], args[fl + 2] = 4, 0           # a flag bit beyond ACCUMULATE | SHIFT_SHARED
        assert fn(*args) == L.SLA_ERR_INVALID and "flags" in L.sla_last_error_string()
        args[fl] = L.SLA_GRAD_ACCUMULATE | L.SLA_GRAD_SHIFT_SHARED
        assert fn(*args) == L.SLA_ERR_INVALID and "plan" in L.sla_last_error_string()
    assert lib.sla_edges_workspace_bytes(None) == 0
    assert lib.sla_edges_destroy(None) == L.SLA_OK


def test_workspace_sizes_grow_with_size():
    a = L.sla_transpose_workspace_bytes(100, 100, 1000)
    b = L.sla_transpose_workspace_bytes(100_000, 100_000, 1_000_000)
    assert 0 < a < b
    assert L.sla_coo_workspace_bytes(10, 10, 100) > 0
    assert L.sla_transpose_workspace_bytes(-1, 1, 1) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "_LIB_PATH", str(tmp_path / "libsla.so"))
    with pytest.raises(ImportError, match="missing"):
        L.lib()


def _header_struct_fields(name):
    """(type, field) pairs of a `typedef struct { ... } name;` in include/sla.h."""
    src = open(os.path.join(ROOT, "include", "sla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    m = re.search(r"typedef struct\s*\{([^}]*)\}\s*" + name + r"\s*;", src)
    assert m, name
    out = []
    for decl in m.group(1).split(";"):
        decl = decl.strip()
        if not decl:
            continue
        parts = decl.split()
        ctype, names = parts[0], " ".join(parts[1:])
        for n in names.split(","):
            n = n.strip().lstrip("*")
            out.append((ctype, n))
    return out


_CTYPES = {"int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64, "double": ctypes.c_double}


@pytest.mark.parametrize("name,mirror", [("sla_csr_props", "sla_csr_props"), ("sla_cg_opts", "sla_cg_opts")])
def test_ctypes_mirrors_match_the_header(name, mirror):
    """Field names, order and types of the binding's structures are the header's,
    so the two sides agree on the layout."""
    hdr = _header_struct_fields(name)
    fields = getattr(L, mirror)._fields_
    assert [n for _, n in hdr] == [f[0] for f in fields]
    for (ct, n), (fn, ft) in zip(hdr, fields):
        assert _CTYPES[ct] == ft, (n, ct, ft)


def test_info_struct_is_three_device_pointers():
    hdr = _header_struct_fields("sla_cg_info")
    assert [n for _, n in hdr] == [f[0] for f in L.sla_cg_info._fields_] == ["iters", "relres", "status"]


def test_list_create_argument_errors_need_no_gpu():
    lib = L.lib()
    h = ctypes.c_void_p()
    assert lib.sla_csr_list_create(0, ctypes.c_void_p(256), 4, 0, ctypes.c_void_p(256), None, 0, 0, None,
                                   ctypes.byref(h)) == L.SLA_ERR_INVALID
    assert "n_items" in L.sla_last_error_string() and h.value is None
    assert lib.sla_csr_list_create(2, None, 4, 0, ctypes.c_void_p(256), None, 0, 0, None,
                                   ctypes.byref(h)) == L.SLA_ERR_INVALID
    assert "item_rows" in L.sla_last_error_string()
    assert lib.sla_csr_list_create(2, ctypes.c_void_p(256), 4, 0, ctypes.c_void_p(256), None, 0, 0, None,
                                   None) == L.SLA_ERR_INVALID


def test_bounds_report_needs_the_bounds_checking_build():
    """The regular library declines the report; the bounds-checking build loads
    without a GPU, exports the same symbols and says what it is."""
    v, c, i = ctypes.c_uint64(7), ctypes.c_int32(7), ctypes.c_int64(7)
    st = L.lib().sla_debug_bounds_report(ctypes.byref(v), ctypes.byref(c), ctypes.byref(i), 0)
    assert st == L.SLA_ERR_UNSUPPORTED and "SLA_DEBUG_BOUNDS" in L.sla_last_error_string()
    assert (v.value, c.value, i.value) == (0, 0, -1)
    path = os.path.join(ROOT, "differentiable_sparse_linear_csr_b200", "libsla_debug_bounds.so")
    if not os.path.exists(path):
        pytest.skip("bounds-checking library not built")
    dbg = ctypes.CDLL(path)
    missing = [n for n in _declared_functions() if not hasattr(dbg, n)]
    assert not missing, missing
    dbg.sla_version.restype = ctypes.c_char_p
    assert b"bounds-checking" in dbg.sla_version()
