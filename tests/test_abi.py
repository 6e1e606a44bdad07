"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/nmspmm.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import structured_sparse_gemm_compress_b200 as nm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nmspmm.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nm_[a-z0-9_]+)\s*\(", text)))


def test_library_builds_and_loads():
    from structured_sparse_gemm_compress_b200 import build
    build.build()
    assert nm.nm_version().startswith("nmspmm")


def test_every_declared_symbol_is_exported():
    declared = declared_functions()
    assert len(declared) >= 10
    out = subprocess.check_output(["nm", "-D", "--defined-only", nm.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    assert sorted(nm.EXPORTS) == declared


def _compress_raw(W_ptr, n_out, k, dt, N, M):
    out = ctypes.c_void_p(123)
    st = nm.lib().nm_compress(W_ptr, n_out, k, dt, N, M, None, ctypes.byref(out))
    return st, out.value


@pytest.mark.parametrize("args,status", [
    ((None, 4, 8, nm.NM_INT8, 2, 4), nm.NM_ERR_INVALID),          # null W
    ((16, 0, 8, nm.NM_INT8, 2, 4), nm.NM_ERR_INVALID),            # n_out = 0
    ((16, 4, -8, nm.NM_INT8, 2, 4), nm.NM_ERR_INVALID),           # k < 0
    ((16, 4, 8, 7, 2, 4), nm.NM_ERR_INVALID),                     # unknown dtype
    ((16, 4, 8, nm.NM_INT8, 3, 4), nm.NM_ERR_UNSUPPORTED),        # 3:4
    ((16, 4, 16, nm.NM_INT8, 1, 8), nm.NM_ERR_UNSUPPORTED),       # 1:8
    ((16, 4, 8, nm.NM_INT8, 5, 4), nm.NM_ERR_INVALID),            # N > M
    ((16, 4, 10, nm.NM_INT8, 2, 4), nm.NM_ERR_INVALID),           # k % M != 0
    ((17, 4, 8, nm.NM_FP16, 2, 4), nm.NM_ERR_INVALID),            # misaligned fp16 W
    ((16, 1 << 25, 8, nm.NM_INT8, 2, 4), nm.NM_ERR_UNSUPPORTED),  # n_out above 2^24
    ((16, 4, (1 << 17) + 4, nm.NM_INT8, 2, 4), nm.NM_ERR_UNSUPPORTED),  # INT8 k: int32 could overflow
])
def test_compress_rejects_before_touching_the_device(args, status):
    st, handle = _compress_raw(*args)
    assert st == status
    assert handle is None  # *out cleared on failure
    assert nm.nm_last_error() != ""


def test_null_handle_paths():
    L = nm.lib()
    assert L.nm_spmm(None, None, 0, None, None, None) == nm.NM_ERR_INVALID
    assert L.nm_decompress(None, None, None) == nm.NM_ERR_INVALID
    assert L.nm_export(None, None, None) == nm.NM_ERR_INVALID
    assert L.nm_query(None, None, None, None, None, None) == nm.NM_ERR_INVALID
    assert L.nm_device_status(None) == nm.NM_ERR_INVALID
    assert L.nm_export_sizes(None, None, None) == nm.NM_ERR_INVALID
    assert L.nm_plan_query(None, 197, 0, None) == nm.NM_ERR_INVALID
    assert L.nm_spmm_noalloc(None, None, 0, None, None, None) == nm.NM_ERR_INVALID
    L.nm_destroy(None)  # no-op


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(nm, "_lib", None)
    monkeypatch.setattr(nm, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        nm.lib()


def test_header_compiles_as_c_and_cpp(tmp_path):
    """include/nmspmm.h is a plain C header: a C99 and a C++11 translation unit
    that take the address of every declared entry point compile cleanly."""
    refs = "\n".join(f"    (void)&{f};" for f in declared_functions())
    src = f'#include "nmspmm.h"\nint main(void) {{\n{refs}\n    return 0;\n}}\n'
    for cc, std, ext in (("gcc", "-std=c99", "c"), ("g++", "-std=c++11", "cpp")):
        path = tmp_path / f"use_header.{ext}"
        path.write_text(src)
        subprocess.check_call([cc, std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                               os.path.dirname(HEADER), "-c", str(path), "-o", str(tmp_path / f"use_{ext}.o")])


@pytest.mark.parametrize("args,status", [
    ((None, 4, 8, nm.NM_INT8, 2, 4), nm.NM_ERR_INVALID),          # null W
    ((16, 4, 8, nm.NM_BF16, 2, 4), nm.NM_ERR_UNSUPPORTED),        # bfloat16 column sums are not exact
    ((16, 4, 8, nm.NM_INT8, 3, 4), nm.NM_ERR_UNSUPPORTED),        # 3:4
    ((16, 4, 10, nm.NM_INT8, 2, 4), nm.NM_ERR_INVALID),           # k % M != 0
    ((17, 4, 8, nm.NM_FP16, 2, 4), nm.NM_ERR_INVALID),            # misaligned fp16 W
])
def test_compress_tile_rejects_before_touching_the_device(args, status):
    out = ctypes.c_void_p(123)
    st = nm.lib().nm_compress_tile(*args, None, ctypes.byref(out))
    assert st == status
    assert out.value is None
    assert nm.nm_last_error() != ""


def test_gather_null_handle_paths():
    L = nm.lib()
    assert L.nm_spmm_gather(None, None, 0, 0, None, None, None) == nm.NM_ERR_INVALID
    assert L.nm_spmm_gather_ex(None, None, 0, 0, None, None, None) == nm.NM_ERR_INVALID
