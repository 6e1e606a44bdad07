"""GPU parity for tile-shared N:M patterns and the activation-gather SpMM.

* nm_compress_tile: canonical format (values + 4-bit positions) bit-exact
  against the oracle's tile-shared compress with 128-row tiles; the masked
  weight decoded from the gather image bit-exact;
* nm_spmm_gather: INT8 (int32, and fp32 with per-channel scale) bit-exact
  against the oracle's GEMM over its masked weight; FP16 within
  max |err| <= 2e-3 * max|Y_ref| and relative Frobenius <= 1e-3 of fp64.
Sizes span several 128-channel tiles, several gather k-blocks with a ragged
kept-k tail, ragged token tiles, and activation row pitches above T.
"""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_gemm_compress_b200 as nm
from structured_sparse_gemm_compress_b200 import inputs

pytestmark = pytest.mark.gpu

PATTERNS = [(1, 4), (2, 4), (2, 8), (4, 8), (4, 4), (8, 8)]


@pytest.fixture(autouse=True)
def _no_forced_plan(monkeypatch):
    for k in ("NMSPMM_FORCE_BN", "NMSPMM_FORCE_SPLITK", "NMSPMM_FORCE_GRID", "NMSPMM_W_BULK", "NMSPMM_GATHER_TMA"):
        monkeypatch.delenv(k, raising=False)


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def _weights(dtype, n_out, K, seed):
    if dtype == "int8":
        return inputs.int8_uniform((n_out, K), -127, 127, seed)
    return inputs.float_normal((n_out, K), 0.02, seed, dtype)


def _acts(dtype, T, K, seed):
    if dtype == "int8":
        return inputs.int8_uniform((T, K), -128, 127, seed)
    return inputs.float_normal((T, K), 1.0, seed, dtype)


def _oracle_masked(W: np.ndarray, N, M):
    v, i = oracle.compress_tile(W, N, M, tile=128)
    return v, i, oracle.decompress(v, i, W.shape[0], W.shape[1], N, M)


def _feature_major(X: torch.Tensor, pad: int) -> torch.Tensor:
    """[k, T] view (rows contiguous) of X^T inside a buffer of row pitch >= T
    with ldx * sizeof(elem) a multiple of 16 bytes, plus `pad` spare columns
    filled with a sentinel that must not leak into Y."""
    T, K = X.shape
    q = 16 // X.element_size()
    ldx = (T + q - 1) // q * q + pad
    buf = torch.full((K, ldx), 77, dtype=X.dtype, device="cuda")
    buf[:, :T] = X.t().cuda()
    return buf[:, :T]


def _assert_float_close(Y_gpu, Y_ref):
    got = Y_gpu.double().cpu().numpy()
    err = np.abs(got - Y_ref)
    mx = np.abs(Y_ref).max()
    assert err.max() <= 2e-3 * mx, (err.max(), mx)
    assert np.linalg.norm(got - Y_ref) <= 1e-3 * np.linalg.norm(Y_ref)


# --------------------------------------------------------------------------- compress


@pytest.mark.parametrize("dtype", ["int8", "fp16"])
@pytest.mark.parametrize("N,M", PATTERNS)
@pytest.mark.parametrize("n_out,K", [(200, 784), (37, 40), (300, 1024), (128, 256)])
def test_compress_tile_bit_exact(dtype, N, M, n_out, K):
    W = _weights(dtype, n_out, K, seed=300 + n_out + K)
    if dtype == "int8":  # many exact ties between column sums
        W = (W // 40).to(torch.int8)
    h = nm.nm_compress_tile(W.cuda(), N, M)
    values, idx = nm.nm_export(h)
    ref_v, ref_i, ref_Wm = _oracle_masked(_np(W), N, M)
    assert np.array_equal(_np(values).view(np.uint8), ref_v.view(np.uint8))
    assert np.array_equal(idx.numpy(), ref_i)
    Wm = nm.nm_decompress(h)
    torch.cuda.synchronize()
    assert np.array_equal(_np(Wm).view(np.uint8), ref_Wm.view(np.uint8))


def test_compress_tile_fp16_scores_exact():
    """A column of 2048 against 2048 plus 127 x 2^-24: an fp32 running sum
    rounds the small terms away and would keep the lower position."""
    W = torch.zeros((128, 8), dtype=torch.float16)
    W[0:2, 0] = 1024.0
    W[0, 1] = 2048.0
    W[1:, 1] = 2.0 ** -24
    W[:, 4] = -1.0
    W[5, 6] = 3.0
    h = nm.nm_compress_tile(W.cuda(), 1, 4)
    values, idx = nm.nm_export(h)
    ref_v, ref_i, _ = _oracle_masked(W.numpy(), 1, 4)
    assert np.array_equal(idx.numpy(), ref_i)
    assert (ref_i[:, 0] & 0xF == 1).all()  # column 1 kept in the first group
    assert np.array_equal(_np(values).view(np.uint16), ref_v.view(np.uint16))


@pytest.mark.parametrize("N,M", [(2, 8), (4, 8)])
def test_recompress_tile_updates_in_place(N, M):
    W1 = _weights("int8", 260, 512, seed=61)
    W2 = _weights("int8", 260, 512, seed=62)
    X = _acts("int8", 90, 512, seed=63)
    h = nm.nm_compress_tile(W1.cuda(), N, M)
    nm.nm_recompress(h, W2.cuda())
    values, idx = nm.nm_export(h)
    ref_v, ref_i, ref_Wm = _oracle_masked(W2.numpy(), N, M)
    assert np.array_equal(values.numpy(), ref_v) and np.array_equal(idx.numpy(), ref_i)
    Y = nm.nm_spmm_gather(h, _feature_major(X, 0))
    assert np.array_equal(Y.cpu().numpy(), oracle.gemm(X.numpy(), ref_Wm))


# --------------------------------------------------------------------------- gather SpMM


@pytest.mark.parametrize("N,M", PATTERNS)
@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("T,n_out,K,pad", [(300, 200, 784, 0), (1, 128, 256, 16), (197, 96, 96, 32),
                                           (64, 384, 3072, 0), (1000, 256, 768, 48)])
def test_spmm_gather_int8_bit_exact(N, M, scaled, T, n_out, K, pad):
    W = _weights("int8", n_out, K, seed=7 + K)
    X = _acts("int8", T, K, seed=8 + T)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=9) if scaled else None
    h = nm.nm_compress_tile(W.cuda(), N, M)
    Y = nm.nm_spmm_gather(h, _feature_major(X, pad), scale=None if s is None else s.cuda())
    _, _, Wm = _oracle_masked(W.numpy(), N, M)
    ref = oracle.gemm(X.numpy(), Wm, scale=None if s is None else s.numpy())
    got = Y.cpu().numpy()
    assert got.dtype == ref.dtype
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("N,M", PATTERNS)
@pytest.mark.parametrize("T,n_out,K", [(300, 200, 392), (5, 256, 1024), (131, 64, 4096)])
def test_spmm_gather_fp16_within_tolerance(N, M, T, n_out, K):
    W = _weights("fp16", n_out, K, seed=17 + K)
    X = _acts("fp16", T, K, seed=18 + T)
    h = nm.nm_compress_tile(W.cuda(), N, M)
    Y = nm.nm_spmm_gather(h, _feature_major(X, 8))
    _, _, Wm = _oracle_masked(_np(W), N, M)
    _assert_float_close(Y, oracle.gemm(_np(X), Wm))


def test_spmm_gather_fp16_scaled():
    W = _weights("fp16", 192, 512, seed=31)
    X = _acts("fp16", 100, 512, seed=32)
    s = inputs.scale_uniform(192, 0.5, 2.0, seed=33)
    h = nm.nm_compress_tile(W.cuda(), 2, 8)
    Y = nm.nm_spmm_gather(h, _feature_major(X, 0), scale=s.cuda())
    _, _, Wm = _oracle_masked(_np(W), 2, 8)
    _assert_float_close(Y, oracle.gemm(_np(X), Wm, scale=s.numpy()))


@pytest.mark.parametrize("bn", ["128", "256"])
@pytest.mark.parametrize("split", ["1", "2", "3"])
@pytest.mark.parametrize("dtype", ["int8", "fp16"])
def test_gather_forced_tiles_and_splits(monkeypatch, bn, split, dtype):
    """The plan (token tile, split-K) must not change INT8 results at all."""
    W = _weights(dtype, 300, 1536, seed=41)
    X = _acts(dtype, 333, 1536, seed=42)
    s = inputs.scale_uniform(300, 0.001, 0.01, seed=43)
    _, _, Wm = _oracle_masked(_np(W), 2, 8)
    monkeypatch.setenv("NMSPMM_FORCE_BN", bn)
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", split)
    h = nm.nm_compress_tile(W.cuda(), 2, 8)
    Xt = _feature_major(X, 0)
    for _ in range(2):  # the second call reuses the re-armed split-K counters
        if dtype == "int8":
            Y = nm.nm_spmm_gather(h, Xt, scale=s.cuda())
            ref = oracle.gemm(X.numpy(), Wm, scale=s.numpy())
            assert np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        else:
            _assert_float_close(nm.nm_spmm_gather(h, Xt), oracle.gemm(_np(X), Wm))
    torch.cuda.synchronize()
    assert nm.nm_device_status(h) == nm.NM_OK


@pytest.mark.parametrize("dtype", ["int8", "fp16"])
@pytest.mark.parametrize("bn", ["128", "256"])
@pytest.mark.parametrize("T,n_out,K", [(300, 200, 784), (1000, 256, 1536), (16, 128, 256)])
def test_gather_tensor_copy_mode(monkeypatch, dtype, bn, T, n_out, K):
    """The alternative gather (four-row tensor copies from the producer warp)
    gives the same results as the default gather warps."""
    W = _weights(dtype, n_out, K, seed=71 + K)
    X = _acts(dtype, T, K, seed=72 + T)
    _, _, Wm = _oracle_masked(_np(W), 2, 8)
    monkeypatch.setenv("NMSPMM_GATHER_TMA", "1")
    monkeypatch.setenv("NMSPMM_FORCE_BN", bn)
    h = nm.nm_compress_tile(W.cuda(), 2, 8)
    Y = nm.nm_spmm_gather(h, _feature_major(X, 16))
    if dtype == "int8":
        assert np.array_equal(Y.cpu().numpy(), oracle.gemm(X.numpy(), Wm))
    else:
        _assert_float_close(Y, oracle.gemm(_np(X), Wm))


@pytest.mark.parametrize("N,M", [(2, 8), (4, 8), (1, 4)])
def test_gather_vit_b_fc2_full_size_sampled(N, M):
    """ViT-B fc2 at T = 12608 in the launch configuration the benchmark uses:
    whole format bit-exact, sampled token rows of Y bit-exact."""
    T, n_out, K = 12608, 768, 3072
    W = _weights("int8", n_out, K, seed=501)
    X = _acts("int8", T, K, seed=502)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=503)
    h = nm.nm_compress_tile(W.cuda(), N, M)
    values, idx = nm.nm_export(h)
    ref_v, ref_i, Wm = _oracle_masked(W.numpy(), N, M)
    assert np.array_equal(values.numpy(), ref_v) and np.array_equal(idx.numpy(), ref_i)
    Y = nm.nm_spmm_gather(h, X.t().contiguous().cuda(), scale=s.cuda())
    rows = np.unique(np.concatenate([np.arange(0, 256), np.arange(T - 200, T),
                                     np.random.default_rng(5).integers(0, T, 300)]))
    ref = oracle.gemm(X.numpy()[rows], Wm, scale=s.numpy())
    assert np.array_equal(Y.cpu().numpy()[rows].view(np.uint32), ref.view(np.uint32))


# --------------------------------------------------------------------------- contract


def test_gather_contract_errors():
    W = _weights("int8", 128, 256, seed=1).cuda()
    X = _acts("int8", 64, 256, seed=2)
    th = nm.nm_compress_tile(W, 2, 4)
    eh = nm.nm_compress(W, 2, 4)
    Xt = _feature_major(X, 0)
    with pytest.raises(nm.NMError) as e:
        nm.nm_spmm(th, X.cuda())
    assert e.value.status == nm.NM_ERR_INVALID
    with pytest.raises(nm.NMError) as e:
        nm.nm_spmm_gather(eh, Xt)
    assert e.value.status == nm.NM_ERR_INVALID
    with pytest.raises(nm.NMError) as e:
        nm.nm_compress_tile(W.to(torch.bfloat16), 2, 4)
    assert e.value.status == nm.NM_ERR_UNSUPPORTED
    with pytest.raises(nm.NMError) as e:
        nm.nm_compress_tile(W, 3, 8)
    assert e.value.status == nm.NM_ERR_UNSUPPORTED
    L = nm.lib()
    Y = torch.empty((64, 128), dtype=torch.int32, device="cuda")
    import ctypes
    st = L.nm_spmm_gather(th.raw, Xt.data_ptr(), 32, 64, Y.data_ptr(), None, None)  # ldx < T
    assert st == nm.NM_ERR_INVALID
    st = L.nm_spmm_gather(th.raw, Xt.data_ptr(), 72, 64, Y.data_ptr(), None, None)  # 72 B pitch
    assert st == nm.NM_ERR_INVALID
    st = L.nm_spmm_gather(th.raw, Xt.data_ptr(), 64, 0, Y.data_ptr(), None, None)   # T = 0: no-op
    assert st == nm.NM_OK
    st = L.nm_spmm_gather(th.raw, Xt.data_ptr(), 64, 64, ctypes.c_void_p(Y.data_ptr() + 4), None, None)
    assert st == nm.NM_ERR_INVALID
    torch.cuda.synchronize()


@pytest.mark.parametrize("N,M", [(1, 4), (2, 8), (4, 8)])
def test_gather_extreme_values_bit_exact(N, M):
    """Largest accumulator magnitudes through the gather: X = -128 everywhere and
    weights at +-127 (every column mass ties, so the tie rule picks every kept k)."""
    n_out, K, T = 256, 4096, 130
    sign = torch.where(inputs.int8_uniform((n_out, K), 0, 1, seed=71) > 0, 127, -127).to(torch.int8)
    sign[:8] = 127
    X = torch.full((T, K), -128, dtype=torch.int8)
    h = nm.nm_compress_tile(sign.cuda(), N, M)
    Y = nm.nm_spmm_gather(h, _feature_major(X, 0))
    _, idx, Wm = _oracle_masked(sign.numpy(), N, M)
    ref = oracle.gemm(X.numpy(), Wm)
    assert np.abs(ref).max() == 128 * 127 * K * N // M
    assert (idx[:, 0] & 0xF == 0).all()  # all masses tie: the lowest positions are kept
    assert np.array_equal(Y.cpu().numpy(), ref)


def test_gather_long_k_and_many_channel_tiles():
    """K = 32768 at 2:8 (K' = 8192: 64 gather k-blocks) and n_out = 20000
    (157 channel tiles, more than the SMs), ragged in both; sampled tokens."""
    for (T, n_out, K, N, M, seed) in ((300, 200, 32768, 2, 8, 91), (70, 20000, 256, 1, 4, 92)):
        W = _weights("int8", n_out, K, seed=seed)
        X = _acts("int8", T, K, seed=seed + 1)
        s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=seed + 2)
        h = nm.nm_compress_tile(W.cuda(), N, M)
        Y = nm.nm_spmm_gather(h, _feature_major(X, 32), scale=s.cuda())
        _, _, Wm = _oracle_masked(W.numpy(), N, M)
        rows = np.unique(np.concatenate([np.arange(0, min(T, 40)), np.arange(max(0, T - 40), T)]))
        ref = oracle.gemm(X.numpy()[rows], Wm, scale=s.numpy())
        assert np.array_equal(Y.cpu().numpy()[rows].view(np.uint32), ref.view(np.uint32))


# --------------------------------------------------------------------------- gather + fused output stage


def _epi_problem(N, M, T=300, n_out=200, K=784):
    W = _weights("int8", n_out, K, seed=401)
    X = _acts("int8", T, K, seed=402)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=403)
    b = inputs.normal_f32((n_out,), 20.0, seed=404)
    _, _, Wm = _oracle_masked(W.numpy(), N, M)
    return W, X, s, b, oracle.gemm(X.numpy(), Wm)


def _as_bits(Y: torch.Tensor) -> np.ndarray:
    Y = Y.cpu()
    if Y.dtype == torch.bfloat16:
        return Y.view(torch.int16).numpy().view(np.uint16)
    return Y.numpy()


@pytest.mark.parametrize("N,M", [(2, 8), (4, 8), (1, 4)])
@pytest.mark.parametrize("out", ["float32", "float16", "bfloat16", "int8"])
def test_gather_ex_outputs_bit_exact(N, M, out):
    """INT8 handle, scale + bias, no activation: every output type bit-exact."""
    W, X, s, b, acc = _epi_problem(N, M)
    os_ = 0.25
    h = nm.nm_compress_tile(W.cuda(), N, M)
    Y = nm.nm_spmm_gather_ex(h, _feature_major(X, 16), scale=s.cuda(), bias=b.cuda(), out=out, out_scale=os_)
    ref = oracle.epilogue(acc, s.numpy(), b.numpy(), "none", out, os_)["exact"]
    assert np.array_equal(_as_bits(Y), ref)


@pytest.mark.parametrize("N,M", [(2, 8), (4, 8)])
def test_gather_ex_int8_gelu_within_bound(N, M):
    """GELU then int8: a code may differ by one only where the oracle's
    unrounded value is within the GELU bound of a half-integer."""
    W, X, s, b, acc = _epi_problem(N, M)
    os_ = 2.0
    h = nm.nm_compress_tile(W.cuda(), N, M)
    Y = nm.nm_spmm_gather_ex(h, _feature_major(X, 0), scale=s.cuda(), bias=b.cuda(), act="gelu", out="int8",
                             out_scale=os_)
    v = oracle.epilogue(acc, s.numpy(), b.numpy(), "none", "float32")["pre"]
    r = oracle.epilogue(acc, s.numpy(), b.numpy(), "gelu", "int8", os_)
    g = r["pre"]
    tol = 4e-7 * np.abs(v) + 2e-6 * np.abs(g) + 1e-30
    q = Y.cpu().numpy().astype(np.int64)
    diff = np.abs(q - r["q"].astype(np.int64))
    assert diff.max() <= 1
    slack = os_ * tol + 2.0 ** -23 * np.abs(r["q_pre"]) + 1e-6
    near = np.abs(np.abs(r["q_pre"] - np.floor(r["q_pre"])) - 0.5) <= slack
    assert np.all(near[diff == 1])
    assert (diff == 0).mean() > 0.999


def test_gather_ex_fp16_handle_and_fixed_routing():
    W = _weights("fp16", 256, 512, seed=411)
    X = _acts("fp16", 150, 512, seed=412)
    b = inputs.normal_f32((256,), 0.5, seed=413)
    h = nm.nm_compress_tile(W.cuda(), 2, 8)
    Xt = _feature_major(X, 8)
    _, _, Wm = _oracle_masked(_np(W), 2, 8)
    acc = oracle.gemm(_np(X), Wm)
    Y = nm.nm_spmm_gather_ex(h, Xt, bias=b.cuda(), out="float32")
    ref = oracle.epilogue(acc, None, b.numpy(), "none", "float32")["pre"]
    err = np.abs(Y.double().cpu().numpy() - ref)
    assert err.max() <= 2e-3 * np.abs(ref).max()
    # no output stage requested: the fixed stage, identical to nm_spmm_gather
    assert torch.equal(nm.nm_spmm_gather_ex(h, Xt), nm.nm_spmm_gather(h, Xt))
    with pytest.raises(nm.NMError):
        nm.nm_spmm_gather_ex(h, Xt, out="int8")   # integer outputs need an INT8 handle
