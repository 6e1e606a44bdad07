"""Failure detection without a GPU fault: the SpMM kernel's waits are bounded.

The test hook leaves one pipeline stage unfilled, so the MMA warp's wait on it
can only run out.  The kernel must then record NM_ERR_TIMEOUT in the handle's
error word, drain its own copies and MMAs, free tensor memory and return; the
CUDA context stays usable and the next normal call is exact again.
"""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_gemm_compress_b200 as nm
from structured_sparse_gemm_compress_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(monkeypatch):
    # one unit of three k-blocks per CTA, so stage #1 of every CTA exists
    monkeypatch.setenv("NMSPMM_FORCE_BN", "128")
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", "1")
    W = inputs.int8_uniform((256, 768), -127, 127, seed=101)
    X = inputs.int8_uniform((256, 768), -128, 127, seed=102)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Xd = X.cuda()
    Y = torch.zeros((256, 256), dtype=torch.int32, device="cuda")
    st = nm.nm_test_spmm_skip_stage(h, Xd, Y, None, skip_stage=1, timeout_ns=50_000_000)
    assert st == nm.NM_OK, nm.nm_last_error()
    torch.cuda.synchronize()  # no CUDA error: the kernel returned on its own
    assert nm.nm_device_status(h) == nm.NM_ERR_TIMEOUT
    assert "bounded wait" in nm.nm_last_error()
    assert nm.nm_device_status(h) == nm.NM_OK  # reading the word clears it
    Y2 = nm.nm_spmm(h, Xd)
    torch.cuda.synchronize()
    assert nm.nm_device_status(h) == nm.NM_OK
    assert np.array_equal(Y2.cpu().numpy(), oracle.spmm(X.numpy(), W.numpy(), 2, 4))


@pytest.mark.parametrize("mode", ["global", "cluster"])
def test_timeout_under_split_k_leaves_the_next_split_call_exact(monkeypatch, mode):
    """k = 1280 in two splits (k-blocks 0-2 and 3-4): skipping stage #2 starves
    only the first split of every tile, so the second split finishes.  In
    global-memory mode it has then counted itself on the tile's arrival
    counter; the next call must not mistake its first arriver for the last
    (the counters are cleared before every split launch).  In cluster mode the
    finished CTA waits at the cluster barrier until its peer gives up."""
    monkeypatch.setenv("NMSPMM_FORCE_BN", "128")
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", "2")
    monkeypatch.setenv("NMSPMM_SPLIT_GLOBAL", "1" if mode == "global" else "0")
    W = inputs.int8_uniform((256, 1280), -127, 127, seed=111)
    X = inputs.int8_uniform((256, 1280), -128, 127, seed=112)
    h = nm.nm_compress(W.cuda(), 2, 4)
    assert nm.nm_plan_query(h, 256)["cluster"] == (1 if mode == "cluster" else 0)
    Xd = X.cuda()
    Y = torch.zeros((256, 256), dtype=torch.int32, device="cuda")
    st = nm.nm_test_spmm_skip_stage(h, Xd, Y, None, skip_stage=2, timeout_ns=50_000_000)
    assert st == nm.NM_OK, nm.nm_last_error()
    torch.cuda.synchronize()
    assert nm.nm_device_status(h) == nm.NM_ERR_TIMEOUT
    ref = oracle.spmm(X.numpy(), W.numpy(), 2, 4)
    for _ in range(2):
        Y2 = nm.nm_spmm(h, Xd)
        torch.cuda.synchronize()
        assert nm.nm_device_status(h) == nm.NM_OK
        assert np.array_equal(Y2.cpu().numpy(), ref)


def test_hook_rejects_bad_timeouts():
    h = nm.nm_compress(inputs.int8_uniform((128, 256), -127, 127, seed=1).cuda(), 2, 4)
    X = torch.zeros((8, 256), dtype=torch.int8, device="cuda")
    Y = torch.zeros((8, 128), dtype=torch.int32, device="cuda")
    assert nm.nm_test_spmm_skip_stage(h, X, Y, None, 0, 0) == nm.NM_ERR_INVALID
    assert nm.nm_test_spmm_skip_stage(h, X, Y, None, 0, 3_000_000_000) == nm.NM_ERR_INVALID
