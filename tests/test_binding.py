"""The Python binding's host-side logic, on CPU: the nm_epilogue struct matches
the header's field order and types, the default output type follows the
header's rule, and every entry point rejects host tensors and bad shapes
before touching a device."""
import ctypes
import os
import re

import pytest
import torch

import structured_sparse_gemm_compress_b200 as nm

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nmspmm.h")


def test_epilogue_struct_matches_the_header():
    text = open(HEADER).read()
    body = re.search(r"typedef struct nm_epilogue \{(.*?)\} nm_epilogue;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = [line.split()[-1].rstrip(";").lstrip("*") for line in body.strip().splitlines() if line.strip()]
    assert fields == [f for f, _ in nm.NMEpilogue._fields_]
    # enum values as the header numbers them
    for name, val in nm.OUT_TYPES.items():
        key = {"default": "DEFAULT", "int32": "INT32", "float32": "FP32", "float16": "FP16",
               "bfloat16": "BF16", "int8": "INT8"}[name]
        assert re.search(rf"NM_OUT_{key}\s*=\s*{val}\b", text), name
    assert re.search(r"NM_ACT_NONE\s*=\s*0", text) and re.search(r"NM_ACT_GELU\s*=\s*1", text)
    assert ctypes.sizeof(nm.NMEpilogue) == 4 + 4 + 8 + 8 + 8  # two enums, two pointers, a float + padding


class _FakeHandle:
    def __init__(self, dtype):
        self.dtype = dtype


@pytest.mark.parametrize("dtype,scale,bias,act,want", [
    (torch.int8, None, None, "none", "int32"),
    (torch.int8, object(), None, "none", "float32"),
    (torch.int8, None, object(), "none", "float32"),
    (torch.int8, None, None, "gelu", "float32"),
    (torch.float16, None, None, "none", "float16"),
    (torch.bfloat16, object(), object(), "gelu", "bfloat16"),
])
def test_default_output_type_rule(dtype, scale, bias, act, want):
    assert nm.resolve_out(_FakeHandle(dtype), "default", scale, bias, act) == want
    assert nm.resolve_out(_FakeHandle(dtype), "int8", scale, bias, act) == "int8"  # explicit wins


def _handle(dtype=torch.int8, tile=False):
    # a handle object whose raw pointer is never reached: every call below fails its checks first
    return nm.NMHandle(0, 256, 768, 2, 4, nm._TORCH_DT[dtype], tile=tile)


def test_entry_points_reject_host_tensors_and_bad_shapes():
    h = _handle()
    X = torch.zeros((16, 768), dtype=torch.int8)                  # host tensor
    with pytest.raises(ValueError):
        nm.nm_compress(X, 2, 4)
    with pytest.raises(ValueError):
        nm.nm_compress_tile(X, 2, 8)
    with pytest.raises(ValueError):
        nm.nm_spmm(h, X)
    with pytest.raises(ValueError):
        nm.nm_spmm_ex(h, X, out="int8")
    with pytest.raises(ValueError):
        nm.nm_spmm_gather(_handle(tile=True), X.t())
    with pytest.raises(ValueError):
        nm.nm_spmm_gather_ex(_handle(tile=True), X.t(), out="int8")


def test_destroyed_handle_refuses_use():
    h = _handle()
    h.destroy()
    with pytest.raises(RuntimeError):
        _ = h.raw
