"""Build libnmspmm.so (sm_100a) in-tree with nvcc.

Usage: python -m structured_sparse_gemm_compress_b200.build [--force] [-v] [--trace]

--trace also builds libnmspmm_trace.so: the same sources compiled with
NM_TRACE, whose SpMM kernels record per-CTA pipeline timestamps into a buffer
named by NMSPMM_TRACE_PTR (see trace.py).  The product library never has them.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")
LIB = os.path.join(PKG, "libnmspmm.so")
TRACE_LIB = os.path.join(PKG, "libnmspmm_trace.so")
OBJDIR = os.path.join(PKG, "_build")
TRACE_OBJDIR = os.path.join(PKG, "_build_trace")
SOURCES = ["nm_api.cu", "nm_pack.cu", "nm_spmm.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", "-I", INCLUDE, "-I", CSRC]


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    deps = [src] + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(INCLUDE, "nmspmm.h"))
    return any(os.path.getmtime(d) > os.path.getmtime(obj) for d in deps)


def _compile(src: str, force: bool, extra: list[str], objdir: str = OBJDIR) -> str:
    obj = os.path.join(objdir, os.path.splitext(src)[0] + ".o")
    path = os.path.join(CSRC, src)
    if force or _stale(obj, path):
        subprocess.check_call([NVCC, *FLAGS, *extra, "-c", path, "-o", obj])
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, trace: bool = False) -> str:
    lib, objdir = (TRACE_LIB, TRACE_OBJDIR) if trace else (LIB, OBJDIR)
    os.makedirs(objdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    if trace:
        extra.append("-DNM_TRACE")
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, extra, objdir), SOURCES))
    if force or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        tmp = lib + f".{os.getpid()}.tmp"
        subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs,
                               "-o", tmp, "-lcudart"])
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
    if "--trace" in sys.argv:
        print(build(force="--force" in sys.argv, trace=True))
