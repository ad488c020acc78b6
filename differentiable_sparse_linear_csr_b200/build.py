"""Builds libsla.so (the sm_100a CUDA library behind include/sla.h) in-tree.

nvcc cross-compiles for sm_100a on a machine without a GPU; each source file is
compiled to an object in parallel (under _build/) and the objects are linked
into one shared library next to this file, so that it travels with the source
tree.  `variant="debug_bounds"` builds libsla_debug_bounds.so with
SLA_DEBUG_BOUNDS defined: every index the kernels read from the pattern is
checked against its range before use (see include/sla.h,
sla_debug_bounds_report).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [*ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC"]
VARIANTS = {"": [], "debug_bounds": ["-DSLA_DEBUG_BOUNDS=1"]}


def lib_path(variant: str = "") -> str:
    return os.path.join(PKG, f"libsla{'_' + variant if variant else ''}.so")


LIB = lib_path()


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def _deps() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(PKG, "csrc", "*.cuh"))) + [
        os.path.join(ROOT, "include", "sla.h")]


def needs_build(variant: str = "") -> bool:
    lib = lib_path(variant)
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          variant: str = "") -> str:
    lib = lib_path(variant)
    if not force and not needs_build(variant):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    objdir = os.path.join(PKG, "_build", variant or "release")
    os.makedirs(objdir, exist_ok=True)
    flags = [*NVCC_FLAGS, *VARIANTS[variant], *(extra or [])]

    def compile_one(src: str) -> str:
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc, *flags, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        return obj

    srcs = sources()
    with ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 1)) as pool:
        objs = list(pool.map(compile_one, srcs))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    v = next((a.split("=", 1)[1] for a in sys.argv if a.startswith("--variant=")), "")
    print(build(force="--force" in sys.argv, verbose=True, variant=v))
