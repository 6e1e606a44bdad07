"""The allocation-free SpMM entry point, checked against nm_spmm through the C ABI.

nm_spmm_noalloc serves callers that cannot allocate device memory (a serving
engine that owns nearly all of HBM through its own pool; latency-critical code
that must not call cudaMalloc/cudaFree, which can synchronise the device).  Its
scratch for a global-memory split-K is a fixed array inside the library instead
of a workspace the handle allocates.  The planner's own plans never need it
(they do not split k, or they reduce the splits on chip), so these tests force
shapes onto the global-memory split-K path so the array is really used, run two
calls in a row (the array keeps the previous call's contents), and compare
every output with the existing entry point: bit-exact for INT8, the FP16
tolerance of the parity suite for FP16.  One test runs the default plans,
which must match nm_spmm as well.  This file is collected last so a failure
here cannot hide the other suites' results.
"""
import ctypes

import numpy as np
import pytest
import torch

import structured_sparse_gemm_compress_b200 as nm
from structured_sparse_gemm_compress_b200 import inputs

pytestmark = pytest.mark.gpu


def _call_noalloc(h, X, Y, scale):
    return nm.lib().nm_spmm_noalloc(h.raw, X.data_ptr(), X.shape[0], Y.data_ptr(),
                                    None if scale is None else scale.data_ptr(),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("split", ["2", "3"])
@pytest.mark.parametrize("N,M,scaled", [(2, 4, True), (1, 4, False), (4, 8, True)])
def test_noalloc_int8_matches_nm_spmm_twice(monkeypatch, split, N, M, scaled):
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", split)
    monkeypatch.setenv("NMSPMM_SPLIT_GLOBAL", "1")
    W = inputs.int8_uniform((768, 768), -127, 127, seed=71).cuda()
    s = inputs.scale_uniform(768, 0.001, 0.01, seed=73).cuda() if scaled else None
    h = nm.nm_compress(W, N, M)
    for call in range(2):
        X = inputs.int8_uniform((197, 768), -128, 127, seed=72 + call).cuda()
        want = nm.nm_spmm(h, X, scale=s)
        got = torch.full_like(want, -1)
        assert _call_noalloc(h, X, got, s) == nm.NM_OK, nm.nm_last_error()
        torch.cuda.synchronize()
        assert nm.nm_device_status(h) == nm.NM_OK
        a, b = got.cpu().numpy(), want.cpu().numpy()
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), f"call {call}"


def test_noalloc_fp16_within_tolerance_twice(monkeypatch):
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", "4")
    monkeypatch.setenv("NMSPMM_SPLIT_GLOBAL", "1")
    W = inputs.float_normal((256, 2048), 0.02, seed=81, dtype="fp16").cuda()
    h = nm.nm_compress(W, 2, 4)
    for call in range(2):
        X = inputs.float_normal((40, 2048), 1.0, seed=82 + call, dtype="fp16").cuda()
        want = nm.nm_spmm(h, X).double()
        got = torch.empty((40, 256), dtype=torch.float16, device="cuda")
        assert _call_noalloc(h, X, got, None) == nm.NM_OK, nm.nm_last_error()
        torch.cuda.synchronize()
        err = (got.double() - want).abs()
        assert err.max().item() <= 2e-3 * want.abs().max().item()
        assert torch.linalg.norm(got.double() - want).item() <= 1e-3 * torch.linalg.norm(want).item()


@pytest.mark.parametrize("T", [197, 12608])
@pytest.mark.parametrize("n_out,K", [(768, 768), (768, 3072)])
def test_noalloc_default_plan_matches_nm_spmm_twice(monkeypatch, T, n_out, K):
    for k in ("NMSPMM_FORCE_SPLITK", "NMSPMM_SPLIT_GLOBAL", "NMSPMM_FORCE_BN"):
        monkeypatch.delenv(k, raising=False)
    W = inputs.int8_uniform((n_out, K), -127, 127, seed=75).cuda()
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=76).cuda()
    h = nm.nm_compress(W, 2, 4)
    for call in range(2):
        X = inputs.int8_uniform((T, K), -128, 127, seed=77 + call).cuda()
        want = nm.nm_spmm(h, X, scale=s)
        got = torch.full_like(want, -1)
        assert _call_noalloc(h, X, got, s) == nm.NM_OK, nm.nm_last_error()
        torch.cuda.synchronize()
        assert nm.nm_device_status(h) == nm.NM_OK
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), f"call {call}"


def test_noalloc_rejects_scratch_beyond_the_limit(monkeypatch):
    monkeypatch.setenv("NMSPMM_FORCE_BN", "128")
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", "3")
    monkeypatch.setenv("NMSPMM_SPLIT_GLOBAL", "1")
    W = inputs.int8_uniform((512, 768), -127, 127, seed=91).cuda()
    X = inputs.int8_uniform((1024, 768), -128, 127, seed=92).cuda()
    h = nm.nm_compress(W, 2, 4)
    Y = torch.empty((1024, 512), dtype=torch.int32, device="cuda")
    # 4 x 8 tiles x 3 splits x 64 KiB = 6 MiB > 4 MiB
    assert _call_noalloc(h, X, Y, None) == nm.NM_ERR_UNSUPPORTED
    assert "static" in nm.nm_last_error() or "holds at most" in nm.nm_last_error()
