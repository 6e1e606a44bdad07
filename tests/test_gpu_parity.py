"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

* compressed format (values + 4-bit positions): bit-exact;
* masked weight decoded from the packed operand image: bit-exact;
* INT8 SpMM (int32, and fp32 with per-channel scale): bit-exact;
* FP16 SpMM: max |err| <= 2e-3 * max|Y_ref| and relative Frobenius error
  <= 1e-3 against the fp64 oracle;
* BF16 SpMM: max |err| <= 4e-3 * max|Y_ref|, relative Frobenius <= 2.5e-3
  (bf16 keeps 8 significant bits: rounding the output once costs up to
  2^-9 = 1.95e-3 relative per element, plus fp32 accumulation error).
Sizes span several 128-channel and token tiles with ragged tails.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import structured_sparse_gemm_compress_b200 as nm
from structured_sparse_gemm_compress_b200 import inputs

pytestmark = pytest.mark.gpu

PATTERNS = [(1, 4), (2, 4), (2, 8), (4, 8), (4, 4), (8, 8)]
TOL = {"fp16": (2e-3, 1e-3), "bf16": (4e-3, 2.5e-3)}
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_4x8.json")


def _np(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _weights(dtype, n_out, K, seed):
    if dtype == "int8":
        return inputs.int8_uniform((n_out, K), -127, 127, seed)
    return inputs.float_normal((n_out, K), 0.02, seed, dtype)


def _acts(dtype, T, K, seed):
    if dtype == "int8":
        return inputs.int8_uniform((T, K), -128, 127, seed)
    return inputs.float_normal((T, K), 1.0, seed, dtype)


def _assert_float_close(Y_gpu: torch.Tensor, Y_ref: np.ndarray, dtype: str):
    got = Y_gpu.double().cpu().numpy()
    err = np.abs(got - Y_ref)
    mx = np.abs(Y_ref).max()
    amax, frob = TOL[dtype]
    assert err.max() <= amax * mx, (err.max(), mx)
    assert np.linalg.norm(got - Y_ref) <= frob * np.linalg.norm(Y_ref)


@pytest.fixture(autouse=True)
def _no_forced_plan(monkeypatch):
    for k in ("NMSPMM_FORCE_BN", "NMSPMM_FORCE_SPLITK", "NMSPMM_FORCE_XS", "NMSPMM_FORCE_GRID",
              "NMSPMM_FORCE_PAIR", "NMSPMM_TMA_STORE", "NMSPMM_SPLIT_GLOBAL", "NMSPMM_CSPLIT",
              "NMSPMM_PREFETCH"):
        monkeypatch.delenv(k, raising=False)


# --------------------------------------------------------------------------- compress / decompress


@pytest.mark.parametrize("dtype", ["int8", "fp16", "bf16"])
@pytest.mark.parametrize("N,M", PATTERNS)
@pytest.mark.parametrize("n_out,K", [(200, 784), (37, 40), (128, 256)])
def test_compress_format_and_image_bit_exact(dtype, N, M, n_out, K):
    W = _weights(dtype, n_out, K, seed=100 + n_out + K)
    if dtype == "int8":  # plenty of exact ties and zeros
        W = (W // 40).to(torch.int8)
    h = nm.nm_compress(W.cuda(), N, M)
    values, idx = nm.nm_export(h)
    ref_v, ref_i = oracle.compress(_np(W, dtype), N, M, dtype)
    assert np.array_equal(_np(values, dtype), ref_v)
    assert np.array_equal(idx.numpy(), ref_i)
    Wm = nm.nm_decompress(h)
    torch.cuda.synchronize()
    ref_Wm = oracle.decompress(ref_v, ref_i, n_out, K, N, M, dtype)
    assert np.array_equal(_np(Wm, dtype), ref_Wm)


@pytest.mark.parametrize("N,M", [(2, 4), (4, 8)])
def test_recompress_updates_in_place(N, M):
    W1 = _weights("int8", 200, 512, seed=61)
    W2 = _weights("int8", 200, 512, seed=62)
    X = _acts("int8", 90, 512, seed=63)
    h = nm.nm_compress(W1.cuda(), N, M)
    nm.nm_recompress(h, W2.cuda())
    values, idx = nm.nm_export(h)
    ref_v, ref_i = oracle.compress(W2.numpy(), N, M)
    assert np.array_equal(values.numpy(), ref_v) and np.array_equal(idx.numpy(), ref_i)
    Y = nm.nm_spmm(h, X.cuda())
    assert np.array_equal(Y.cpu().numpy(), oracle.spmm(X.numpy(), W2.numpy(), N, M))


def test_hand_examples_on_gpu():
    g = json.load(open(GOLDEN))
    W = torch.zeros((4, 16), dtype=torch.int8)
    X = torch.zeros((2, 16), dtype=torch.int8)
    W[:, :8] = torch.tensor(g["W"], dtype=torch.int8)   # zero groups appended: Y is unchanged
    X[:, :8] = torch.tensor(g["X"], dtype=torch.int8)
    for nm_str, case in g["cases"].items():
        N, M = map(int, nm_str.split(":"))
        h = nm.nm_compress(W.cuda(), N, M)
        Y = nm.nm_spmm(h, X.cuda())
        assert Y.cpu().tolist() == case["Y"], nm_str


# --------------------------------------------------------------------------- SpMM parity


@pytest.mark.parametrize("N,M", PATTERNS)
@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("T,n_out,K", [(300, 200, 784), (1, 128, 256), (197, 96, 96), (64, 384, 3072)])
@pytest.mark.parametrize("tma_store", ["0", "1"])
def test_spmm_int8_bit_exact(monkeypatch, N, M, scaled, T, n_out, K, tma_store):
    monkeypatch.setenv("NMSPMM_TMA_STORE", tma_store)
    W = _weights("int8", n_out, K, seed=7 + K)
    X = _acts("int8", T, K, seed=8 + T)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=9) if scaled else None
    h = nm.nm_compress(W.cuda(), N, M)
    Y = nm.nm_spmm(h, X.cuda(), scale=None if s is None else s.cuda())
    ref = oracle.spmm(X.numpy(), W.numpy(), N, M, scale=None if s is None else s.numpy())
    got = Y.cpu().numpy()
    assert got.dtype == ref.dtype
    if scaled:
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    else:
        assert np.array_equal(got, ref)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("N,M", PATTERNS)
@pytest.mark.parametrize("T,n_out,K", [(300, 200, 392), (5, 256, 1024), (131, 64, 4096)])
@pytest.mark.parametrize("tma_store", ["0", "1"])
def test_spmm_float_within_tolerance(monkeypatch, dtype, N, M, T, n_out, K, tma_store):
    monkeypatch.setenv("NMSPMM_TMA_STORE", tma_store)
    W = _weights(dtype, n_out, K, seed=17 + K)
    X = _acts(dtype, T, K, seed=18 + T)
    h = nm.nm_compress(W.cuda(), N, M)
    Y = nm.nm_spmm(h, X.cuda())
    ref = oracle.spmm(_np(X, dtype), _np(W, dtype), N, M, dtype=dtype)
    _assert_float_close(Y, ref, dtype)


def test_spmm_fp16_scaled():
    W = _weights("fp16", 192, 512, seed=31)
    X = _acts("fp16", 100, 512, seed=32)
    s = inputs.scale_uniform(192, 0.5, 2.0, seed=33)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda())
    ref = oracle.spmm(_np(X, "fp16"), _np(W, "fp16"), 2, 4, scale=s.numpy(), dtype="fp16")
    _assert_float_close(Y, ref, "fp16")


@pytest.mark.parametrize("mode", ["cluster", "global"])
@pytest.mark.parametrize("bn", ["32", "64", "128", "192"])
@pytest.mark.parametrize("split", ["1", "2", "3", "5"])
def test_forced_tiles_and_splits_are_bit_identical(monkeypatch, bn, split, mode):
    """Adaptive parallelism must not change INT8 results at all: every token
    tile and split, with the partials reduced on chip (cluster) or in global
    memory (workspace and arrival counters)."""
    W = _weights("int8", 200, 1280, seed=41)
    X = _acts("int8", 150, 1280, seed=42)
    s = inputs.scale_uniform(200, 0.001, 0.01, seed=43)
    ref = oracle.spmm(X.numpy(), W.numpy(), 2, 4, scale=s.numpy())
    monkeypatch.setenv("NMSPMM_FORCE_BN", bn)
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", split)
    monkeypatch.setenv("NMSPMM_SPLIT_GLOBAL", "1" if mode == "global" else "0")
    h = nm.nm_compress(W.cuda(), 2, 4)
    plan = nm.nm_plan_query(h, 150, scaled=True)
    assert plan["splits"] == int(split) and plan["bn"] == int(bn)
    assert plan["cluster"] == (1 if (mode == "cluster" and split != "1") else 0)
    for _ in range(2):  # the second call reuses the workspace and its counters
        Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda())
        assert np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("S", [2, 3, 4, 8])
@pytest.mark.parametrize("bn", ["32", "64", "128"])
@pytest.mark.parametrize("n_out", [200, 198])
@pytest.mark.parametrize("N,M", [(2, 4), (4, 8)])
def test_cluster_split_int8_outputs_bit_exact(monkeypatch, S, bn, n_out, N, M):
    """On-chip split-K: int32 and scaled fp32 outputs, whole (n_out % 4 == 0,
    16-byte stores) and ragged (element stores) channel groups, ragged T."""
    K, T = 2048, 197
    W = _weights("int8", n_out, K, seed=401 + n_out)
    X = _acts("int8", T, K, seed=402)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=403)
    monkeypatch.setenv("NMSPMM_FORCE_BN", bn)
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", str(S))
    h = nm.nm_compress(W.cuda(), N, M)
    assert nm.nm_plan_query(h, T)["cluster"] == 1
    for scaled in (False, True):
        Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda() if scaled else None)
        torch.cuda.synchronize()
        assert nm.nm_device_status(h) == nm.NM_OK
        ref = oracle.spmm(X.numpy(), W.numpy(), N, M, scale=s.numpy() if scaled else None)
        assert np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("S", [2, 4, 8])
@pytest.mark.parametrize("n_out", [256, 190])
def test_cluster_split_float_within_tolerance(monkeypatch, dtype, S, n_out):
    K, T = 2048, 77
    W = _weights(dtype, n_out, K, seed=411)
    X = _acts(dtype, T, K, seed=412)
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", str(S))
    h = nm.nm_compress(W.cuda(), 2, 4)
    assert nm.nm_plan_query(h, T)["cluster"] == 1
    Y = nm.nm_spmm(h, X.cuda())
    torch.cuda.synchronize()
    assert nm.nm_device_status(h) == nm.NM_OK
    _assert_float_close(Y, oracle.spmm(_np(X, dtype), _np(W, dtype), 2, 4, dtype=dtype), dtype)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_cluster_split_runtime_output_stage_float(monkeypatch, dtype):
    """nm_spmm_ex on an FP16/BF16 handle under the on-chip split: scale, bias
    and GELU, fp32 output, within the float tolerance of the fp64 oracle."""
    K, T, n_out = 2048, 61, 190
    W = _weights(dtype, n_out, K, seed=441)
    X = _acts(dtype, T, K, seed=442)
    s = inputs.scale_uniform(n_out, 0.5, 2.0, seed=443)
    b = inputs.scale_uniform(n_out, -1.0, 1.0, seed=444)
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", "4")
    h = nm.nm_compress(W.cuda(), 2, 4)
    assert nm.nm_plan_query(h, T, scaled=True)["cluster"] == 1
    Y = nm.nm_spmm_ex(h, X.cuda(), scale=s.cuda(), bias=b.cuda(), act="gelu", out="float32")
    torch.cuda.synchronize()
    ref = oracle.spmm_epilogue(_np(X, dtype), _np(W, dtype), 2, 4, scale=s.numpy(), bias=b.numpy(), act="gelu",
                               out="float32", dtype=dtype)["pre"]
    got = Y.double().cpu().numpy()
    amax, frob = TOL[dtype]
    assert np.abs(got - ref).max() <= amax * np.abs(ref).max()
    assert np.linalg.norm(got - ref) <= frob * np.linalg.norm(ref)


def test_cluster_split_runtime_output_stage_bit_exact(monkeypatch):
    """nm_spmm_ex under the on-chip split: scale, bias and int8 requantisation."""
    K, T, n_out = 3072, 197, 198
    W = _weights("int8", n_out, K, seed=421)
    X = _acts("int8", T, K, seed=422)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=423)
    b = inputs.scale_uniform(n_out, -2.0, 2.0, seed=424)
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", "6")
    h = nm.nm_compress(W.cuda(), 2, 4)
    assert nm.nm_plan_query(h, T, scaled=True)["cluster"] == 1
    for out in ("int8", "float32"):
        Y = nm.nm_spmm_ex(h, X.cuda(), scale=s.cuda(), bias=b.cuda(), out=out, out_scale=0.05)
        torch.cuda.synchronize()
        ref = oracle.spmm_epilogue(X.numpy(), W.numpy(), 2, 4, scale=s.numpy(), bias=b.numpy(), out=out,
                                   out_scale=0.05)
        assert np.array_equal(Y.cpu().numpy(), ref["exact"]), out


@pytest.mark.parametrize("N,M", [(2, 4), (4, 8)])
@pytest.mark.parametrize("n_out,K", [(768, 768), (2304, 768), (3072, 768), (768, 3072)])
def test_planner_splits_small_token_counts_on_chip(n_out, K, N, M):
    """At a few tokens the unsplit tiles of the long-k ViT-B layer (fc2, 12
    k-blocks on 6 to 12 CTAs) leave almost every SM idle: the planner splits k
    over a cluster.  The 3-k-block layers are not split (the on-chip reduction
    costs more than their k loop), and at T = 12608 nothing is split.  Whatever
    the plan, the result is the oracle's."""
    W = _weights("int8", n_out, K, seed=431)
    h = nm.nm_compress(W.cuda(), N, M)
    big = nm.nm_plan_query(h, 12608, scaled=True)
    assert big["splits"] == 1 and big["cluster"] == 0
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=433)
    for T in (16, 64, 197):
        small = nm.nm_plan_query(h, T, scaled=True)
        if K == 3072 and T <= 64:
            assert small["splits"] > 1 and small["cluster"] == 1, (T, small)
        if K == 768:
            assert small["splits"] == 1, (T, small)
        if small["splits"] > 1:
            assert small["cluster"] == 1 and small["grid"] == small["units"]
        X = _acts("int8", T, K, seed=432 + T)
        Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda())
        ref = oracle.spmm(X.numpy(), W.numpy(), N, M, scale=s.numpy())
        assert np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32)), T


@pytest.mark.parametrize("dtype,K,n_out,T,want", [
    ("int8", 768, 768, 12608, 1),     # 6 channel tiles, 3 x 99 pair tiles
    ("int8", 768, 2304, 12608, 1),
    ("int8", 768, 384, 12608, 0),     # 3 channel tiles: the last pair would compute a padding tile
    ("int8", 768, 576, 100352, 0),    # 5 channel tiles
    ("int8", 768, 192, 12608, 0),     # 1 x 99 pair tiles, fewer than the SMs
    ("int8", 768, 768, 6272, None),   # 3 x 49 = 147 pair tiles: pair iff the GPU has <= 147 SMs
    ("int8", 96, 768, 100352, 0),     # under 192 bytes of X per token
    ("int8", 3072, 384, 12608, 1),    # >= 2 KB of X per token: pair whatever the tile count
    ("fp16", 768, 768, 6304, 1),      # 1536 bytes per token, 3 x 50 pair tiles
])
def test_planner_pair_rule(dtype, K, n_out, T, want):
    """The planner takes the two-SM kernel when its 256-channel tiles are whole
    (an even count of 128-channel tiles) and there are at least as many 256 x
    128 pair tiles as SMs (K*b >= 192 bytes), or when a token row of X is at
    least 2 KB."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if want is None:
        want = int(3 * 49 >= sms)
    h = nm.nm_compress(_weights(dtype, n_out, K, seed=441).cuda(), 2, 4)
    assert nm.nm_plan_query(h, T, scaled=True)["pair"] == want


@pytest.mark.parametrize("n_out,want_pair", [(256, 1), (384, 0), (250, 1)])
def test_planner_pair_rule_parity(monkeypatch, n_out, want_pair):
    """The same rule on a GPU capped at 16 persistent CTAs (16 pair tiles are
    enough), and the output of whichever kernel it picks is the oracle's."""
    monkeypatch.setenv("NMSPMM_FORCE_GRID", "16")
    T, K = 2000, 768
    W = _weights("int8", n_out, K, seed=451)
    X = _acts("int8", T, K, seed=452)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=453)
    h = nm.nm_compress(W.cuda(), 2, 4)
    assert nm.nm_plan_query(h, T, scaled=True)["pair"] == want_pair
    Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda())
    ref = oracle.spmm(X.numpy(), W.numpy(), 2, 4, scale=s.numpy())
    assert np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("grid", ["5", "148"])
@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (2, 8), (4, 8), (4, 4)])
@pytest.mark.parametrize("T,n_out,K", [(1000, 300, 768), (129, 200, 512), (640, 384, 256)])
@pytest.mark.parametrize("tma_store", ["0", "1"])
def test_x_stationary_bit_exact(monkeypatch, grid, N, M, T, n_out, K, tma_store):
    """X tile resident across the channel tiles of a CTA's range (token-tile switches included)."""
    monkeypatch.setenv("NMSPMM_TMA_STORE", tma_store)
    W = _weights("int8", n_out, K, seed=201 + K)
    X = _acts("int8", T, K, seed=202 + T)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=203)
    monkeypatch.setenv("NMSPMM_FORCE_XS", "1")
    monkeypatch.setenv("NMSPMM_FORCE_PAIR", "0")
    monkeypatch.setenv("NMSPMM_FORCE_GRID", grid)
    h = nm.nm_compress(W.cuda(), N, M)
    for scaled in (True, False):
        Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda() if scaled else None)
        torch.cuda.synchronize()
        assert nm.nm_device_status(h) == nm.NM_OK
        ref = oracle.spmm(X.numpy(), W.numpy(), N, M, scale=s.numpy() if scaled else None)
        assert np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("bn", ["128", "192", "224"])
@pytest.mark.parametrize("grid", ["6", "148"])
@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (2, 8), (4, 8), (8, 8)])
@pytest.mark.parametrize("T,n_out,K", [(1000, 300, 768), (130, 640, 512), (450, 256, 1280)])
@pytest.mark.parametrize("tma_store", ["0", "1"])
def test_cta_pair_bit_exact(monkeypatch, bn, grid, N, M, T, n_out, K, tma_store):
    """CTA-pair kernel: ragged T, odd channel-tile counts (n_out=300), several tiles per pair."""
    monkeypatch.setenv("NMSPMM_TMA_STORE", tma_store)
    W = _weights("int8", n_out, K, seed=301 + K)
    X = _acts("int8", T, K, seed=302 + T)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=303)
    monkeypatch.setenv("NMSPMM_FORCE_PAIR", "1")
    monkeypatch.setenv("NMSPMM_FORCE_BN", bn)
    monkeypatch.setenv("NMSPMM_FORCE_GRID", grid)
    h = nm.nm_compress(W.cuda(), N, M)
    for scaled in (True, False):
        Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda() if scaled else None)
        torch.cuda.synchronize()
        assert nm.nm_device_status(h) == nm.NM_OK
        ref = oracle.spmm(X.numpy(), W.numpy(), N, M, scale=s.numpy() if scaled else None)
        assert np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("tma_store", ["0", "1", "runtime-stage"])
def test_cta_pair_repeated_calls_few_clusters(monkeypatch, tma_store):
    """Accumulator hand-over between the two CTAs of a pair under load: six
    clusters walk 12 tiles each, so every accumulator is released and refilled
    six times per call; 30 calls, alternating scaled and unscaled outputs (the
    fixed stages: fp32 and int32; the runtime stage: fp32 with a zero bias),
    must all be bit-exact and end without a timed-out wait."""
    runtime = tma_store == "runtime-stage"  # the output stage read from the launch (nm_spmm_ex)
    monkeypatch.setenv("NMSPMM_TMA_STORE", "0" if runtime else tma_store)
    monkeypatch.setenv("NMSPMM_FORCE_PAIR", "1")
    monkeypatch.setenv("NMSPMM_FORCE_BN", "128")
    monkeypatch.setenv("NMSPMM_FORCE_GRID", "12")
    T, n_out, K = 4500, 512, 768  # 2 channel-tile pairs x 36 token tiles = 72 pair tiles
    W = _weights("int8", n_out, K, seed=461)
    X = _acts("int8", T, K, seed=462)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=463)
    refs = {True: oracle.spmm(X.numpy(), W.numpy(), 2, 4, scale=s.numpy()),
            False: oracle.spmm(X.numpy(), W.numpy(), 2, 4)}
    h = nm.nm_compress(W.cuda(), 2, 4)
    plan = nm.nm_plan_query(h, T, scaled=True)
    assert plan["pair"] == 1 and plan["grid"] == 6
    Xd, sd = X.cuda(), s.cuda()
    zero = torch.zeros(n_out, dtype=torch.float32, device="cuda")
    bad = []
    for i in range(30):
        scaled = i % 2 == 0
        if runtime:  # a (zero) bias routes the call to the runtime stage; fp32 out with and without the scale
            Y = nm.nm_spmm_ex(h, Xd, scale=sd if scaled else None, bias=zero, out="float32")
            ref = refs[scaled] if scaled else refs[False].astype(np.float32)
            torch.cuda.synchronize()
            assert nm.nm_device_status(h) == nm.NM_OK, i
            if not np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32)):
                bad.append(i)
            continue
        Y = nm.nm_spmm(h, Xd, scale=sd if scaled else None)
        torch.cuda.synchronize()
        assert nm.nm_device_status(h) == nm.NM_OK, i
        if not np.array_equal(Y.cpu().numpy().view(np.uint32), refs[scaled].view(np.uint32)):
            bad.append(i)
    assert not bad, bad


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("bn", ["128", "224"])
@pytest.mark.parametrize("N,M", [(2, 4), (2, 8), (4, 8)])
def test_cta_pair_float_within_tolerance(monkeypatch, dtype, bn, N, M):
    W = _weights(dtype, 384, 1024, seed=311)
    X = _acts(dtype, 500, 1024, seed=312)
    monkeypatch.setenv("NMSPMM_FORCE_PAIR", "1")
    monkeypatch.setenv("NMSPMM_FORCE_BN", bn)
    h = nm.nm_compress(W.cuda(), N, M)
    Y = nm.nm_spmm(h, X.cuda())
    torch.cuda.synchronize()
    assert nm.nm_device_status(h) == nm.NM_OK
    _assert_float_close(Y, oracle.spmm(_np(X, dtype), _np(W, dtype), N, M, dtype=dtype), dtype)


@pytest.mark.parametrize("grid", ["3", "11"])
def test_streaming_mode_many_units_per_cta(monkeypatch, grid):
    W = _weights("int8", 300, 1024, seed=211)
    X = _acts("int8", 700, 1024, seed=212)
    monkeypatch.setenv("NMSPMM_FORCE_XS", "0")
    monkeypatch.setenv("NMSPMM_FORCE_PAIR", "0")
    monkeypatch.setenv("NMSPMM_FORCE_GRID", grid)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Y = nm.nm_spmm(h, X.cuda())
    assert np.array_equal(Y.cpu().numpy(), oracle.spmm(X.numpy(), W.numpy(), 2, 4))


@pytest.mark.parametrize("mode", ["cluster", "global"])
@pytest.mark.parametrize("split", ["1", "4"])
def test_forced_split_fp16_within_tolerance(monkeypatch, split, mode):
    W = _weights("fp16", 256, 2048, seed=51)
    X = _acts("fp16", 40, 2048, seed=52)
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", split)
    monkeypatch.setenv("NMSPMM_SPLIT_GLOBAL", "1" if mode == "global" else "0")
    h = nm.nm_compress(W.cuda(), 2, 8)
    Y = nm.nm_spmm(h, X.cuda())
    _assert_float_close(Y, oracle.spmm(_np(X, "fp16"), _np(W, "fp16"), 2, 8, dtype="fp16"), "fp16")


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("bn", ["64", "192"])
def test_forced_tile_float_within_tolerance(monkeypatch, dtype, bn):
    W = _weights(dtype, 300, 1024, seed=61)
    X = _acts(dtype, 700, 1024, seed=62)
    monkeypatch.setenv("NMSPMM_FORCE_BN", bn)
    monkeypatch.setenv("NMSPMM_FORCE_PAIR", "0")
    h = nm.nm_compress(W.cuda(), 2, 4)
    Y = nm.nm_spmm(h, X.cuda())
    _assert_float_close(Y, oracle.spmm(_np(X, dtype), _np(W, dtype), 2, 4, dtype=dtype), dtype)


# --------------------------------------------------------------------------- full-size workloads (sampled)


def _sampled_rows(T, count, seed, h=None, scaled=False):
    """Random rows plus, when the handle is given, the first and last token of
    every token tile of the plan the call uses (every half tile for the two-SM
    kernel, whose CTAs each hold half of the tile's tokens), so that every
    (channel tile, token tile) pair the kernel writes is compared: all
    columns of each row are checked."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(T, size=min(count, T), replace=False).tolist())
    rows.update({0, T - 1})
    if h is not None:
        plan = nm.nm_plan_query(h, T, scaled=scaled)
        step = plan["bn"] // 2 if plan["pair"] else plan["bn"]
        for t0 in range(0, T, step):
            rows.update({t0, min(t0 + step, T) - 1})
    return np.array(sorted(rows))


@pytest.mark.parametrize("layer", inputs.single_layer(), ids=lambda l: l.name)
def test_single_layer_full(layer):
    W, X = layer.weight(), layer.activation()
    h = nm.nm_compress(W.cuda(), layer.N, layer.M)
    Y = nm.nm_spmm(h, X.cuda())
    assert np.array_equal(Y.cpu().numpy(), oracle.spmm(X.numpy(), W.numpy(), layer.N, layer.M))


@pytest.mark.parametrize("layer", inputs.vit_b_int8(), ids=lambda l: f"{l.name}-{l.nm}")
def test_vit_b_int8_sampled_rows(layer):
    W, X, s = layer.weight(), layer.activation(), layer.scale()
    h = nm.nm_compress(W.cuda(), layer.N, layer.M)
    Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda())
    rows = _sampled_rows(layer.T, 48, layer.seed, h, scaled=True)
    ref = oracle.spmm(X.numpy()[rows], W.numpy(), layer.N, layer.M, scale=s.numpy())
    assert np.array_equal(Y.cpu().numpy()[rows].view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("layer", inputs.vit_l_fp16(), ids=lambda l: f"{l.name}-{l.nm}")
def test_vit_l_fp16_sampled_rows(layer):
    W, X = layer.weight(), layer.activation()
    h = nm.nm_compress(W.cuda(), layer.N, layer.M)
    Y = nm.nm_spmm(h, X.cuda())
    rows = _sampled_rows(layer.T, 32, layer.seed, h)
    ref = oracle.spmm(_np(X, "fp16")[rows], _np(W, "fp16"), layer.N, layer.M, dtype="fp16")
    _assert_float_close(Y[rows.tolist()], ref, "fp16")


@pytest.mark.parametrize("layer", inputs.swin_t_int8(), ids=lambda l: f"{l.name}-{l.nm}")
def test_swin_t_int8_sampled_rows(layer):
    W, X, s = layer.weight(), layer.activation(), layer.scale()
    h = nm.nm_compress(W.cuda(), layer.N, layer.M)
    Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda())
    rows = _sampled_rows(layer.T, 48, layer.seed, h, scaled=True)
    ref = oracle.spmm(X.numpy()[rows], W.numpy(), layer.N, layer.M, scale=s.numpy())
    assert np.array_equal(Y.cpu().numpy()[rows].view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("T", [197, 50432])
def test_vit_b_mixed_sequence(T):
    """All 48 layers back to back in one stream; every layer checked (sampled rows at large T)."""
    layers = inputs.vit_b_mixed(T)
    outs = []
    for l in layers:
        W, X, s = l.weight(), l.activation(), l.scale()
        h = nm.nm_compress(W.cuda(), l.N, l.M)
        outs.append((l, X, W, s, h, nm.nm_spmm(h, X.cuda(), scale=s.cuda())))
    torch.cuda.synchronize()
    for l, X, W, s, h, Y in outs:
        rows = _sampled_rows(l.T, 16, l.seed, h, scaled=True) if T > 1000 else np.arange(T)
        ref = oracle.spmm(X.numpy()[rows], W.numpy(), l.N, l.M, scale=s.numpy())
        assert np.array_equal(Y.cpu().numpy()[rows].view(np.uint32), ref.view(np.uint32)), l.name


# --------------------------------------------------------------------------- edge cases and errors


@pytest.mark.parametrize("N,M", [(2, 4), (4, 8), (8, 8)])
def test_extreme_values_bit_exact(N, M):
    """Largest accumulator magnitudes: X = -128 everywhere, W at +-127 (and
    ties everywhere, so the tie rule decides every kept position)."""
    n_out, K, T = 256, 4096, 130
    sign = torch.where(inputs.int8_uniform((n_out, K), 0, 1, seed=71) > 0, 127, -127).to(torch.int8)
    sign[:8] = 127    # rows whose every kept product is -128 * 127
    sign[8:16] = -127
    X = torch.full((T, K), -128, dtype=torch.int8)
    h = nm.nm_compress(sign.cuda(), N, M)
    Y = nm.nm_spmm(h, X.cuda())
    ref = oracle.spmm(X.numpy(), sign.numpy(), N, M)
    assert np.abs(ref).max() == 128 * 127 * K * N // M  # the largest magnitude the shape allows
    assert np.array_equal(Y.cpu().numpy(), ref)


def test_long_k_and_many_channel_tiles():
    """K = 16384 (64 k-blocks, CTA-pair kernel) and n_out = 20000 (157 channel
    tiles, more than the SMs), ragged in both."""
    for (T, n_out, K, seed) in ((130, 200, 16384, 81), (70, 20000, 256, 82)):
        W = _weights("int8", n_out, K, seed=seed)
        X = _acts("int8", T, K, seed=seed + 1)
        s = inputs.scale_uniform(n_out, 0.001, 0.01, seed=seed + 2)
        h = nm.nm_compress(W.cuda(), 2, 4)
        Y = nm.nm_spmm(h, X.cuda(), scale=s.cuda())
        ref = oracle.spmm(X.numpy(), W.numpy(), 2, 4, scale=s.numpy())
        assert np.array_equal(Y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_t_zero_is_noop():
    h = nm.nm_compress(_weights("int8", 64, 64, 1).cuda(), 2, 4)
    X = torch.empty((0, 64), dtype=torch.int8, device="cuda")
    Y = nm.nm_spmm(h, X)
    assert Y.shape == (0, 64)


def test_spmm_rejects_unaligned_and_unsupported():
    h = nm.nm_compress(_weights("int8", 64, 64, 1).cuda(), 2, 4)
    buf = torch.zeros(64 * 64 + 16, dtype=torch.int8, device="cuda")
    Y = torch.empty((64, 64), dtype=torch.int32, device="cuda")
    L = nm.lib()
    assert L.nm_spmm(h.raw, buf.data_ptr() + 1, 64, Y.data_ptr(), None, None) == nm.NM_ERR_INVALID
    assert L.nm_spmm(h.raw, buf.data_ptr(), -1, Y.data_ptr(), None, None) == nm.NM_ERR_INVALID
    h8 = nm.nm_compress(_weights("int8", 16, 8, 1).cuda(), 2, 4)  # k = 8 bytes per row: not TMA-able
    assert L.nm_spmm(h8.raw, buf.data_ptr(), 4, Y.data_ptr(), None, None) == nm.NM_ERR_UNSUPPORTED
    assert "multiple of 16" in nm.nm_last_error()


def test_output_canaries_untouched():
    """Ragged tiles must not write past Y (guard elements after the output)."""
    W = _weights("int8", 200, 784, 3)
    X = _acts("int8", 77, 784, 4)
    h = nm.nm_compress(W.cuda(), 2, 4)
    buf = torch.full((77 * 200 + 4096,), -7, dtype=torch.int32, device="cuda")
    Y = buf[: 77 * 200].view(77, 200)
    nm.nm_spmm(h, X.cuda(), Y=Y)
    assert (buf[77 * 200:] == -7).all()
    assert np.array_equal(Y.cpu().numpy(), oracle.spmm(X.numpy(), W.numpy(), 2, 4))
