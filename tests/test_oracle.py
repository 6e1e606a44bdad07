"""Pins for the CPU oracle, checked against what the paper and mathematics fix.

Each pin is independent of the oracle's own code: hand-worked examples
(tests/golden), brute-force subset enumeration, numpy's integer / float64
matmul over an independently built mask, exact decoders checked against
numpy / torch conversions, and structural invariants.  A dropped term, a wrong
sign, a wrong tie rule or a transposed operand in the oracle fails at least one.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_4x8.json")
PATTERNS = [(1, 4), (2, 4), (2, 8), (4, 8)]


def _kept_pairs(values, idx, N, M, k):
    """Decode (value, position) pairs per row from the canonical format."""
    rows = []
    for r in range(values.shape[0]):
        flat_v = values[r].reshape(-1)
        pairs = []
        for e in range(len(flat_v)):
            b = idx[r, e // 2]
            p = (b >> 4) if (e & 1) else (b & 0xF)
            pairs.append((flat_v[e].item(), int(p)))
        rows.append(pairs)
    return rows


def _brute_force_keep(mags, N):
    """Best N-subset: maximal sum of |w|, then lexicographically smallest positions."""
    best = None
    for sub in itertools.combinations(range(len(mags)), N):
        key = (-sum(mags[p] for p in sub), sub)
        if best is None or key < best:
            best = key
    return list(best[1])


def _numpy_mask(W, N, M):
    """Independent top-N mask: stable argsort of -|w| per group."""
    n, k = W.shape
    a = np.abs(W.astype(np.float64)).reshape(n, k // M, M)
    order = np.argsort(-a, axis=2, kind="stable")[:, :, :N]
    mask = np.zeros_like(a, dtype=bool)
    np.put_along_axis(mask, order, True, axis=2)
    return mask.reshape(n, k)


# --------------------------------------------------------------------------- golden


@pytest.mark.parametrize("nm", ["1:4", "2:4", "2:8", "4:8"])
def test_hand_examples(nm):
    g = json.load(open(GOLDEN))
    N, M = map(int, nm.split(":"))
    W = np.array(g["W"], dtype=np.int8)
    X = np.array(g["X"], dtype=np.int8)
    values, idx = oracle.compress(W, N, M)
    got = _kept_pairs(values, idx, N, M, W.shape[1])
    want = [[tuple(p) for p in row] for row in g["cases"][nm]["kept"]]
    assert got == want
    Y = oracle.spmm(X, W, N, M)
    assert Y.dtype == np.int32
    assert Y.tolist() == g["cases"][nm]["Y"]


@pytest.mark.parametrize("nm", ["1:4", "2:4", "2:8", "4:8"])
def test_hand_examples_match_brute_force(nm):
    """The stored hand-worked kept sets agree with brute-force enumeration."""
    g = json.load(open(GOLDEN))
    N, M = map(int, nm.split(":"))
    for r, row in enumerate(g["W"]):
        want = []
        for gi in range(len(row) // M):
            grp = row[gi * M:(gi + 1) * M]
            for p in _brute_force_keep([abs(v) for v in grp], N):
                want.append((grp[p], p))
        assert [tuple(p) for p in g["cases"][nm]["kept"][r]] == want


# --------------------------------------------------------------------------- compress


@pytest.mark.parametrize("N,M", PATTERNS)
def test_compress_brute_force_int8(N, M):
    rng = np.random.default_rng(11)
    W = rng.integers(-3, 4, size=(24, 8 * M), dtype=np.int8)  # many ties and zeros
    values, idx = oracle.compress(W, N, M)
    got = _kept_pairs(values, idx, N, M, W.shape[1])
    for r in range(W.shape[0]):
        want = []
        for gi in range(W.shape[1] // M):
            grp = W[r, gi * M:(gi + 1) * M].astype(int).tolist()
            for p in _brute_force_keep([abs(v) for v in grp], N):
                want.append((grp[p], p))
        assert got[r] == want


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("N,M", PATTERNS)
def test_compress_brute_force_float(N, M, dtype):
    rng = np.random.default_rng(12)
    base = rng.choice([0.0, -0.0, 0.5, -0.5, 1.0, -1.0, 1.5, 2.0, -2.0, 3.0e-5, -6.0e-8],
                      size=(16, 4 * M))
    t = torch.tensor(base, dtype=torch.float32)
    if dtype == "fp16":
        W = t.to(torch.float16).numpy()
        mags = np.abs(W.astype(np.float64))
    else:
        tb = t.to(torch.bfloat16)
        W = tb.view(torch.int16).numpy().view(np.uint16)
        mags = np.abs(tb.to(torch.float64).numpy())
    values, idx = oracle.compress(W, N, M, dtype)
    pos = _kept_pairs(values, idx, N, M, W.shape[1])
    for r in range(W.shape[0]):
        want = []
        for gi in range(W.shape[1] // M):
            want += [gi * M + p for p in _brute_force_keep(list(mags[r, gi * M:(gi + 1) * M]), N)]
        got = [gi * M + p for gi, (_, p) in zip(np.repeat(np.arange(W.shape[1] // M), N), pos[r])]
        assert got == want
        # stored values are the original bit patterns at those positions
        assert [v for v, _ in pos[r]] == [W[r, c].item() for c in want]


@pytest.mark.parametrize("N,M", PATTERNS + [(4, 4), (8, 8)])
def test_compress_invariants(N, M):
    rng = np.random.default_rng(13)
    W = rng.integers(-127, 128, size=(33, 16 * M), dtype=np.int8)
    values, idx = oracle.compress(W, N, M)
    Wm = oracle.decompress(values, idx, *W.shape, N, M)
    n, k = W.shape
    g = Wm.reshape(n, k // M, M)
    assert ((g != 0).sum(axis=2) <= N).all()
    # decompress(compress(W)) == W masked by an independently computed top-N mask
    assert np.array_equal(Wm, np.where(_numpy_mask(W, N, M), W, 0))
    # positions strictly ascending inside every group
    pairs = _kept_pairs(values, idx, N, M, k)
    for row in pairs:
        for gi in range(k // M):
            ps = [p for _, p in row[gi * N:(gi + 1) * N]]
            assert ps == sorted(set(ps))
    # every kept element beats every dropped one in the (|w| desc, pos asc) order
    mask = _numpy_mask(W, N, M).reshape(n, k // M, M)
    a = np.abs(W.astype(int)).reshape(n, k // M, M)
    for r in range(0, n, 7):
        for gi in range(k // M):
            kept = [p for p in range(M) if mask[r, gi, p]]
            drop = [p for p in range(M) if not mask[r, gi, p]]
            for p in kept:
                for q in drop:
                    assert a[r, gi, p] > a[r, gi, q] or (a[r, gi, p] == a[r, gi, q] and p < q)
    # idempotence
    v2, i2 = oracle.compress(Wm, N, M)
    assert np.array_equal(oracle.decompress(v2, i2, n, k, N, M), Wm)
    if N == M:
        assert np.array_equal(Wm, W)


def test_compress_all_zero_keeps_lowest_positions():
    W = np.zeros((3, 16), dtype=np.int8)
    for N, M in PATTERNS:
        values, idx = oracle.compress(W, N, M)
        pairs = _kept_pairs(values, idx, N, M, 16)
        for row in pairs:
            assert [p for _, p in row] == list(range(N)) * (16 // M)
            assert all(v == 0 for v, _ in row)


def test_idx_layout_odd_count_rows_padded():
    # 1:4 with k = 12 keeps 3 elements per row: 2 bytes per row, high nibble of byte 1 zero.
    W = np.array([[0, 0, 0, 9, 0, 7, 0, 0, 1, 0, 0, 0]] * 2, dtype=np.int8)
    values, idx = oracle.compress(W, 1, 4)
    assert idx.shape == (2, 2)
    assert idx.tolist() == [[0x13, 0x00], [0x13, 0x00]]
    assert values.reshape(2, -1).tolist() == [[9, 7, 1], [9, 7, 1]]


def test_compress_rejects_bad_arguments():
    W = np.zeros((2, 10), dtype=np.int8)
    with pytest.raises(ValueError):
        oracle.compress(W, 2, 4)  # k % M != 0
    with pytest.raises(ValueError):
        oracle.compress(np.zeros((2, 8), dtype=np.int8), 5, 4)  # N > M


# --------------------------------------------------------------------------- GEMM


@pytest.mark.parametrize("N,M", PATTERNS + [(4, 4)])
def test_gemm_int8_matches_numpy_int64(N, M):
    rng = np.random.default_rng(21)
    W = rng.integers(-127, 128, size=(40, 96), dtype=np.int8)
    X = rng.integers(-128, 128, size=(37, 96), dtype=np.int8)
    Y = oracle.spmm(X, W, N, M)
    Wm = np.where(_numpy_mask(W, N, M), W, 0).astype(np.int64)
    assert np.array_equal(Y.astype(np.int64), X.astype(np.int64) @ Wm.T)


def test_gemm_int8_extreme_values_fit_int32():
    X = np.full((2, 4096), -128, dtype=np.int8)
    W = np.full((3, 4096), -128, dtype=np.int8)
    Y = oracle.spmm(X, W, 4, 4)
    assert (Y == 128 * 128 * 4096).all()


def test_gemm_int8_scaled_single_rounding():
    rng = np.random.default_rng(22)
    W = rng.integers(-127, 128, size=(24, 64), dtype=np.int8)
    X = rng.integers(-128, 128, size=(9, 64), dtype=np.int8)
    s = rng.uniform(0.001, 0.01, size=24).astype(np.float32)
    Y = oracle.spmm(X, W, 2, 4, scale=s)
    acc = X.astype(np.int64) @ np.where(_numpy_mask(W, 2, 4), W, 0).astype(np.int64).T
    want = acc.astype(np.int32).astype(np.float32) * s[None, :]  # numpy: one fp32 rounding
    assert Y.dtype == np.float32
    assert np.array_equal(Y.view(np.uint32), want.astype(np.float32).view(np.uint32))


def test_gemm_identity_and_one_hot():
    rng = np.random.default_rng(23)
    W = rng.integers(-127, 128, size=(12, 32), dtype=np.int8)
    Wm = oracle.decompress(*oracle.compress(W, 2, 4), 12, 32, 2, 4)
    eye = np.eye(32, dtype=np.int8)
    assert np.array_equal(oracle.gemm(eye, Wm), Wm.T.astype(np.int32))  # rows of Wm^T
    onehot = np.zeros((1, 32), dtype=np.int8)
    onehot[0, 5] = 1
    assert np.array_equal(oracle.gemm(onehot, Wm)[0], Wm[:, 5].astype(np.int32))


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_gemm_float_matches_numpy_float64(dtype):
    g = torch.Generator().manual_seed(5)
    W = torch.randn(20, 64, generator=g) * 0.02
    X = torch.randn(11, 64, generator=g)
    s = torch.rand(20, generator=g) * 0.01 + 0.001
    if dtype == "fp16":
        Wn, Xn = W.half().numpy(), X.half().numpy()
        Wd, Xd = W.half().double().numpy(), X.half().double().numpy()
    else:
        Wn = W.bfloat16().view(torch.int16).numpy().view(np.uint16)
        Xn = X.bfloat16().view(torch.int16).numpy().view(np.uint16)
        Wd, Xd = W.bfloat16().double().numpy(), X.bfloat16().double().numpy()
    Y = oracle.spmm(Xn, Wn, 2, 4, scale=s.numpy(), dtype=dtype)
    mask = _numpy_mask(Wd, 2, 4)
    want = (Xd @ np.where(mask, Wd, 0.0).T) * s.numpy().astype(np.float64)[None, :]
    assert Y.dtype == np.float64
    np.testing.assert_allclose(Y, want, rtol=1e-12, atol=1e-15)


def test_fp16_decoder_all_finite_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = ((bits >> 10) & 0x1F) != 31
    W = bits[finite].reshape(-1, 1).copy()
    one = np.array([[1.0]], dtype=np.float16).view(np.uint16)
    Y = oracle.gemm(one, W, dtype="fp16")[0]
    assert np.array_equal(Y, W.view(np.float16).astype(np.float64)[:, 0])


def test_bf16_decoder_all_finite_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    W = bits[finite].reshape(-1, 1).copy()
    one = torch.tensor([[1.0]]).bfloat16().view(torch.int16).numpy().view(np.uint16)
    Y = oracle.gemm(one, W, dtype="bf16")[0]
    want = torch.from_numpy(W[:, 0].view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    assert np.array_equal(Y, want)


# ------------------------------------------------------------------ fused output stage

def _golden_epilogue():
    with open(os.path.join(os.path.dirname(__file__), "golden", "epilogue_hand.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden_epilogue()["cases"], ids=lambda c: c["name"])
def test_epilogue_hand_cases(case):
    sc = None if case["scale"] is None else np.array(case["scale"], dtype=np.float32)
    bi = None if case["bias"] is None else np.array(case["bias"], dtype=np.float32)
    exp = np.array(case["expected"])
    if case.get("path") == "float":  # fp64 accumulator of the FP16/BF16 path, compared in fp64
        acc = np.array(case["acc"], dtype=np.float64)
        r = oracle.epilogue(acc, sc, bi, case["act"], case["out"], case["out_scale"])
        assert np.all(np.abs(r["pre"] - exp) <= case["rel_tol"] * np.abs(exp)), (r["pre"], exp)
        return
    acc = np.array(case["acc"], dtype=np.int32)
    if "out_scale_per_case" in case:  # one column at a time, each with its own output scale
        for j, os_ in enumerate(case["out_scale_per_case"]):
            r = oracle.epilogue(acc[:, j:j + 1], None if sc is None else sc[j:j + 1],
                                None if bi is None else bi[j:j + 1], case["act"], case["out"], os_)
            assert int(r["q"][0, 0]) == int(exp[0, j])
        return
    r = oracle.epilogue(acc, sc, bi, case["act"], case["out"], case["out_scale"])
    if case["out"] == "int8":
        assert np.array_equal(r["q"], exp.astype(np.int8))
        assert np.array_equal(r["exact"], exp.astype(np.int8))
    else:
        assert np.array_equal(r["exact"], exp.astype(np.float32))


def test_gelu_matches_normal_cdf_table():
    g = _golden_epilogue()["normal_cdf"]
    for x, phi in zip(g["x"], g["phi"]):
        assert abs(oracle.gelu(x) - x * phi) <= 1e-15 * x
        assert abs(oracle.gelu(-x) - (-x * (1.0 - phi))) <= 1e-15 * x
    assert oracle.gelu(0.0) == 0.0


def test_gelu_odd_part_is_identity():
    # erf is odd, so GELU(x) - GELU(-x) = x/2 (1 + erf) + x/2 (1 - erf) = x
    for x in np.linspace(-8, 8, 161):
        assert abs((oracle.gelu(x) - oracle.gelu(-x)) - x) <= 4e-16 * max(1.0, abs(x))
    # far tails: GELU(x) -> x and GELU(-x) -> 0
    assert oracle.gelu(12.0) == 12.0 and abs(oracle.gelu(-12.0)) < 1e-30


def test_epilogue_int8_saturating_cast_closed_form():
    rng = np.random.default_rng(3)
    acc = rng.integers(-400, 400, size=(7, 33), dtype=np.int64).astype(np.int32)
    r = oracle.epilogue(acc, out="int8")
    assert np.array_equal(r["q"], np.clip(acc, -128, 127).astype(np.int8))
    b = rng.integers(-50, 50, size=33).astype(np.float32)  # integer biases: exact sums
    r = oracle.epilogue(acc, bias=b, out="int8")
    assert np.array_equal(r["q"], np.clip(acc + b.astype(np.int64), -128, 127).astype(np.int8))


def test_epilogue_per_channel_indexing():
    # scale and bias are per output channel (column), never per token (row)
    acc = np.arange(12, dtype=np.int32).reshape(3, 4)
    sc = np.array([1, 2, 4, 8], dtype=np.float32)
    bi = np.array([0, 100, 200, 300], dtype=np.float32)
    r = oracle.epilogue(acc, sc, bi, out="float32")
    want = np.array([[acc[t, n] * 2 ** n + 100 * n for n in range(4)] for t in range(3)], dtype=np.float32)
    assert np.array_equal(r["exact"], want)
    rf = oracle.epilogue(acc.astype(np.float64), sc, bi)
    assert np.array_equal(rf["pre"], want.astype(np.float64))


def test_epilogue_narrow_float_outputs_round_to_nearest_even():
    # fp16 spacing is 2 in [2048, 4096): 2049 is halfway between 2048 and 2050 -> 2048 (even
    # significand), 2051 between 2050 and 2052 -> 2052; 257 and 259 are exact.
    # bf16 spacing is 16 at 2048 and 2 in [256, 512): 2049, 2051 -> 2048; 257 (halfway between
    # 256 and 258) -> 256; 259 (halfway between 258 and 260) -> 260.
    acc = np.array([[2049, 2051, 257, 259]], dtype=np.int32)
    h = oracle.epilogue(acc, out="float16")["exact"]
    assert h.tolist() == [[2048.0, 2052.0, 257.0, 259.0]]
    b = oracle.epilogue(acc, out="bfloat16")["exact"]
    vals = (b.astype(np.uint32) << 16).view(np.float32)
    assert vals.tolist() == [[2048.0, 2048.0, 256.0, 260.0]]


def test_epilogue_rejects_bad_arguments():
    acc = np.zeros((2, 2), dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.epilogue(acc, act="relu")
    with pytest.raises(ValueError):
        oracle.epilogue(acc.astype(np.float64), out="int8")
