"""The allocation-free solve across CUDA contexts of one device (run as a script).

Callers that cannot allocate while they solve often own their contexts: a
runtime may create its own context with the driver API next to the primary one
that the CUDA runtime uses, or reset the device between jobs.  The library's
module, and with it the static scratch array of sla_cg_solve_noalloc, is loaded
into each context at its own address, so the entry point must look the address
up in the context that is current at the call.  This script drives one device
through the driver API (ctypes on libcuda, no PyTorch CUDA use): in the primary
context, in a context it creates, back in the primary context, and in a second
created context, it runs sla_cg_solve with a workspace and then
sla_cg_solve_noalloc twice, and checks that both allocation-free calls match
the regular solve.  It exits 0 when every comparison holds.
"""
import ctypes
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
os.environ["SLA_GRID_ONCHIP"] = "0"   # the handle runs the same grid variant as the no-alloc path

from differentiable_sparse_linear_csr_b200 import _lib as L          # noqa: E402
from differentiable_sparse_linear_csr_b200 import workloads as W     # noqa: E402

cu = ctypes.CDLL("libcuda.so.1")
lib = L.lib()


def ck(r, what):
    if r != 0:
        raise RuntimeError(f"{what} returned {r}")


class Dev:
    """Device buffers of the current context, freed together."""

    def __init__(self):
        self.ptrs = []

    def alloc(self, nbytes):
        p = ctypes.c_uint64()
        ck(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(max(int(nbytes), 256))), "cuMemAlloc")
        self.ptrs.append(p.value)
        return p.value

    def put(self, arr):
        arr = np.ascontiguousarray(arr)
        p = self.alloc(arr.nbytes)
        ck(cu.cuMemcpyHtoD_v2(ctypes.c_uint64(p), arr.ctypes.data_as(ctypes.c_void_p),
                              ctypes.c_size_t(arr.nbytes)), "cuMemcpyHtoD")
        return p

    def get(self, p, shape, dtype):
        out = np.empty(shape, dtype)
        ck(cu.cuMemcpyDtoH_v2(out.ctypes.data_as(ctypes.c_void_p), ctypes.c_uint64(p),
                              ctypes.c_size_t(out.nbytes)), "cuMemcpyDtoH")
        return out

    def free(self):
        for p in self.ptrs:
            cu.cuMemFree_v2(ctypes.c_uint64(p))
        self.ptrs = []


def check_in_current_context(label):
    rp, ci, v = W.poisson2d(150)
    n, nnz = rp.shape[0] - 1, ci.shape[0]
    b = W.normal(3, W.STREAM_B, n)
    d = Dev()
    try:
        rpd, cid, vd, bd = d.put(rp), d.put(ci), d.put(v), d.put(b)
        h = ctypes.c_void_p()
        st = lib.sla_csr_create(n, n, nnz, rpd, cid, 1, L.SLA_F64, L.SLA_FLAG_SYMMETRIC, None,
                                ctypes.byref(h))
        ck(st, "sla_csr_create: " + lib.sla_last_error_string().decode())
        opts = L.make_opts(fixed_iters=120, strategy=L.SLA_STRATEGY_GRID)

        def info():
            it, rr, stt = d.alloc(4), d.alloc(8), d.alloc(4)
            return (it, stt), L.sla_cg_info(it, rr, stt)

        wsb = lib.sla_workspace_bytes(h, L.SLA_OP_CG)
        ws = d.alloc(wsb)
        xr = d.alloc(8 * n)
        ref_ptrs, ref_info = info()
        ck(lib.sla_cg_solve(h, vd, bd, xr, ctypes.byref(opts), ref_info, ws, wsb, None), "sla_cg_solve")
        results = []
        for call in range(2):
            x = d.put(np.full(n, np.nan))
            ptrs, inf = info()
            st = lib.sla_cg_solve_noalloc(n, nnz, rpd, cid, 1, L.SLA_F64, vd, bd, x, ctypes.byref(opts),
                                          inf, None)
            ck(st, "sla_cg_solve_noalloc: " + lib.sla_last_error_string().decode())
            results.append((x, ptrs))
        ck(cu.cuCtxSynchronize(), "cuCtxSynchronize")
        x_ref = d.get(xr, n, np.float64)
        it_ref = int(d.get(ref_ptrs[0], 1, np.int32)[0])
        st_ref = int(d.get(ref_ptrs[1], 1, np.int32)[0])
        for call, (x, ptrs) in enumerate(results):
            xv = d.get(x, n, np.float64)
            it = int(d.get(ptrs[0], 1, np.int32)[0])
            stv = int(d.get(ptrs[1], 1, np.int32)[0])
            err = float(np.linalg.norm(xv - x_ref) / np.linalg.norm(x_ref))
            print(f"{label} call {call}: iters {it}/{it_ref} status {stv}/{st_ref} rel {err:.2e}")
            if not (it == it_ref == 120 and stv == st_ref == L.SLA_FIXED_DONE and err < 1e-8):
                raise AssertionError(f"{label}: allocation-free call {call} differs from sla_cg_solve")
        ck(lib.sla_csr_destroy(h), "sla_csr_destroy")
    finally:
        d.free()


def main():
    ck(cu.cuInit(0), "cuInit")
    dev = ctypes.c_int()
    ck(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
    primary = ctypes.c_void_p()
    ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), dev), "cuDevicePrimaryCtxRetain")
    ck(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
    check_in_current_context("primary context")
    for k in range(2):
        ctx = ctypes.c_void_p()
        ck(cu.cuCtxCreate_v2(ctypes.byref(ctx), 0, dev), "cuCtxCreate")   # becomes current
        try:
            check_in_current_context(f"created context {k}")
        finally:
            ck(cu.cuCtxSynchronize(), "cuCtxSynchronize")
            ck(cu.cuCtxDestroy_v2(ctx), "cuCtxDestroy")
        ck(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
        check_in_current_context(f"primary context again ({k})")
    ck(cu.cuDevicePrimaryCtxRelease_v2(dev), "cuDevicePrimaryCtxRelease")
    print("noalloc contexts: ok")


if __name__ == "__main__":
    main()
