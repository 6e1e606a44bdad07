"""GPU parity of the fused output stage (nm_spmm_ex) against the CPU oracle.

The output stage is the library's own definition (the paper stops at the MMA):
y = act((float)acc * scale[n] + bias[n]) in fp32, one rounding per step, then
fp32 / fp16 / bf16 (round to nearest even) or int8 (round half to even of
y * out_scale, saturated).

* INT8 handle, no activation: every output type is bit-exact.
* GELU: the kernel evaluates erf by Abramowitz and Stegun's formula 7.1.26
  (absolute error at most 1.5e-7) with the hardware's approximate reciprocal
  and power of two, the oracle in fp64, so results agree within
      |y - g| <= 4e-7 |v| + 2e-6 |g|   (v the value before GELU, g = GELU(v))
  plus the output type's own rounding; an int8 code may differ by one only
  where the oracle's unrounded value lies that close to a half-integer.
* FP16/BF16 handles: fp32 accumulation in any order, so the same tolerances
  as the plain SpMM (max |err| <= 2e-3 max|ref|, rel. Frobenius <= 1e-3; bf16
  4e-3 / 2.5e-3), against the fp64 oracle.
Sizes span several token and channel tiles with ragged tails.
"""
import ctypes
import functools

import numpy as np
import pytest
import torch

import oracle
import structured_sparse_gemm_compress_b200 as nm
from structured_sparse_gemm_compress_b200 import inputs

pytestmark = pytest.mark.gpu

T0, K0, N0 = 300, 768, 320   # INT8 case: 3 token tiles (ragged), 3 channel tiles (ragged)
OUTS = ["float32", "float16", "bfloat16", "int8"]


@pytest.fixture(autouse=True)
def _no_forced_plan(monkeypatch):
    for k in ("NMSPMM_FORCE_BN", "NMSPMM_FORCE_SPLITK", "NMSPMM_FORCE_XS", "NMSPMM_FORCE_GRID",
              "NMSPMM_FORCE_PAIR", "NMSPMM_TMA_STORE"):
        monkeypatch.delenv(k, raising=False)


@functools.lru_cache(maxsize=None)
def _int8_problem(N, M, T=T0, K=K0, n_out=N0, seed=7):
    W = inputs.int8_uniform((n_out, K), -127, 127, seed)
    X = inputs.int8_uniform((T, K), -128, 127, seed + 1)
    s = inputs.scale_uniform(n_out, 0.001, 0.01, seed + 2)
    b = inputs.normal_f32((n_out,), 20.0, seed + 3)
    vals, idx = oracle.compress(W.numpy(), N, M)
    Wm = oracle.decompress(vals, idx, n_out, K, N, M)
    acc = oracle.gemm(X.numpy(), Wm)
    return W, X, s, b, acc


def _gpu_np(Y: torch.Tensor) -> np.ndarray:
    Y = Y.cpu()
    if Y.dtype == torch.bfloat16:
        return Y.view(torch.int16).numpy().view(np.uint16)
    return Y.numpy()


def _as_f64(Y: torch.Tensor) -> np.ndarray:
    return Y.double().cpu().numpy()


def _out_scale(scaled: bool) -> float:
    # int8 codes that use the whole range and saturate at both ends
    return 0.25 if scaled else 2e-3


@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (2, 8), (4, 8)])
@pytest.mark.parametrize("out", OUTS)
@pytest.mark.parametrize("scaled,biased", [(False, False), (True, False), (False, True), (True, True)])
def test_int8_output_stage_bit_exact(N, M, out, scaled, biased):
    W, X, s, b, acc = _int8_problem(N, M)
    sc, bi = (s if scaled else None), (b if biased else None)
    os_ = _out_scale(scaled)
    h = nm.nm_compress(W.cuda(), N, M)
    Y = nm.nm_spmm_ex(h, X.cuda(), scale=None if sc is None else sc.cuda(),
                      bias=None if bi is None else bi.cuda(), out=out, out_scale=os_)
    torch.cuda.synchronize()
    ref = oracle.epilogue(acc, None if sc is None else sc.numpy(), None if bi is None else bi.numpy(),
                          "none", out, os_)
    assert np.array_equal(_gpu_np(Y), ref["exact"])
    if out == "int8":  # the case really exercises saturation on both sides
        q = ref["exact"]
        assert (q == 127).any() and (q == -128).any() and ((q > -128) & (q < 127)).mean() > 0.3


@pytest.mark.parametrize("out,os_", [("float32", 1.0), ("int8", 2.0 ** -24), ("int8", 2.0 ** -21)])
def test_output_stage_conversions_at_extreme_accumulators(out, os_):
    """The runtime stage's int32 -> fp32 conversion (rounded to nearest even)
    and int8 rounding across the whole accumulator range: k = 2^17, rows of
    all +127 / all -127 / random signs against X of -128 or random values, so
    |acc| spans the exact range below 2^24, the rounded range above it, and
    reaches 128 * 127 * 2^17 (just under 2^31).  Scale 1 and a zero bias keep
    the value the conversion itself; bit-exact against the oracle."""
    n_out, K, T = 128, 1 << 17, 33
    sign = torch.where(inputs.int8_uniform((n_out, K), 0, 1, seed=91) > 0, 127, -127).to(torch.int8)
    sign[:8] = 127
    sign[8:16] = -127
    for r in range(16, n_out):  # a run of equal signs of growing length: |acc| from 2^20 to 2^27
        sign[r, : 64 * r] = 127 if r % 2 else -127
    X = inputs.int8_uniform((T, K), -128, 127, seed=92)
    X[:8] = -128
    h = nm.nm_compress(sign.cuda(), 4, 4)
    one = torch.ones(n_out, dtype=torch.float32)
    zero = torch.zeros(n_out, dtype=torch.float32)
    Y = nm.nm_spmm_ex(h, X.cuda(), scale=one.cuda(), bias=zero.cuda(), out=out, out_scale=os_)
    torch.cuda.synchronize()
    acc = oracle.gemm(X.numpy(), sign.numpy())
    assert np.abs(acc.astype(np.int64)).max() == 128 * 127 * K
    mag = np.abs(acc.astype(np.int64))
    assert (mag > 2 ** 24).mean() > 0.2 and (mag < 2 ** 22).mean() > 0.2
    ref = oracle.epilogue(acc, one.numpy(), zero.numpy(), "none", out, os_)
    assert np.array_equal(_gpu_np(Y), ref["exact"])


def _gelu_tol(v: np.ndarray, g: np.ndarray) -> np.ndarray:
    return 4e-7 * np.abs(v) + 2e-6 * np.abs(g) + 1e-30


@pytest.mark.parametrize("N,M", [(2, 4), (4, 8)])
@pytest.mark.parametrize("out", OUTS)
def test_int8_gelu_within_erf_bound(N, M, out):
    W, X, s, b, acc = _int8_problem(N, M)
    os_ = 2.0
    h = nm.nm_compress(W.cuda(), N, M)
    Y = nm.nm_spmm_ex(h, X.cuda(), scale=s.cuda(), bias=b.cuda(), act="gelu", out=out, out_scale=os_)
    torch.cuda.synchronize()
    v = oracle.epilogue(acc, s.numpy(), b.numpy(), "none", "float32")["pre"]
    r = oracle.epilogue(acc, s.numpy(), b.numpy(), "gelu", out, os_)
    g = r["pre"]
    tol = _gelu_tol(v, g)
    if out == "int8":
        q = Y.cpu().numpy().astype(np.int64)
        qr = r["q"].astype(np.int64)
        diff = np.abs(q - qr)
        assert diff.max() <= 1
        # the kernel also rounds y * out_scale to fp32 once before rounding to an integer
        slack = os_ * tol + 2.0 ** -23 * np.abs(r["q_pre"]) + 1e-6
        near = np.abs(np.abs(r["q_pre"] - np.floor(r["q_pre"])) - 0.5) <= slack
        assert np.all(near[diff == 1]), "an int8 code differs away from a rounding boundary"
        assert (diff == 0).mean() > 0.999
        assert (qr == 127).any() and (qr == 0).any()
    else:
        got = _as_f64(Y)
        rnd = {"float32": 2.0 ** -24, "float16": 2.0 ** -11, "bfloat16": 2.0 ** -8}[out]
        bound = tol * (1 + rnd) + rnd * np.abs(g) + (6e-8 if out == "float16" else 0.0)
        assert np.all(np.abs(got - g) <= bound), float(np.max(np.abs(got - g) - bound))


def test_gelu_sweep_within_bound():
    """Dense sweep of the GELU input over [-9, 9] (an FP16 handle with one-hot
    activations makes every pre-activation a chosen value): the kernel's fp32
    GELU against the fp64 oracle within the stated bound."""
    n_out, K = 512, 128
    grid = np.linspace(-9.0, 9.0, n_out * K).reshape(n_out, K)
    W = torch.tensor(grid, dtype=torch.float32).to(torch.float16)
    b = torch.tensor(np.linspace(0, 4e-3, n_out), dtype=torch.float32)  # off the fp16 grid
    X = torch.eye(K, dtype=torch.float16)                               # token t picks weight column t
    h = nm.nm_compress(W.cuda(), 4, 4)
    Y = nm.nm_spmm_ex(h, X.cuda(), bias=b.cuda(), act="gelu", out="float32")
    torch.cuda.synchronize()
    acc = W.t().double().numpy()                                        # [T = K, n_out]: exact products
    v = oracle.epilogue(acc, None, b.numpy(), "none", "float32")["pre"]
    g = oracle.epilogue(acc, None, b.numpy(), "gelu", "float32")["pre"]
    got = _as_f64(Y)
    err = np.abs(got - g)
    bound = _gelu_tol(v, g) * (1 + 2.0 ** -24) + 2.0 ** -24 * np.abs(g)
    worst = float(np.max(err - bound))
    print(f"gelu sweep: max |err| {err.max():.3e}, max |err|/|v| {np.max(err / np.maximum(np.abs(v), 1e-30)):.3e}, "
          f"excess over bound {worst:.3e}")
    assert worst <= 0.0


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("out", ["float32", "float16", "bfloat16"])
@pytest.mark.parametrize("act", ["none", "gelu"])
def test_float_handles_output_stage(dtype, out, act):
    T, K, n_out = 200, 512, 200
    W = inputs.float_normal((n_out, K), 0.02, 31, dtype)
    X = inputs.float_normal((T, K), 1.0, 32, dtype)
    s = inputs.scale_uniform(n_out, 0.5, 2.0, 33)
    b = inputs.normal_f32((n_out,), 0.5, 34)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Y = nm.nm_spmm_ex(h, X.cuda(), scale=s.cuda(), bias=b.cuda(), act=act, out=out)
    torch.cuda.synchronize()
    as_np = (lambda t: t.numpy()) if dtype == "fp16" else (lambda t: t.view(torch.int16).numpy().view(np.uint16))
    vals, idx = oracle.compress(as_np(W), 2, 4, dtype)
    Wm = oracle.decompress(vals, idx, n_out, K, 2, 4, dtype)
    acc = oracle.gemm(as_np(X), Wm, None, dtype)
    ref = oracle.epilogue(acc, s.numpy(), b.numpy(), act, out)["pre"]
    amax, frob = (4e-3, 2.5e-3) if "bfloat16" in (out,) or dtype == "bf16" else (2e-3, 1e-3)
    got = _as_f64(Y)
    assert np.abs(got - ref).max() <= amax * np.abs(ref).max()
    assert np.linalg.norm(got - ref) <= frob * np.linalg.norm(ref)


@pytest.mark.parametrize("plan", [
    {"NMSPMM_FORCE_BN": "32"}, {"NMSPMM_FORCE_BN": "64"}, {"NMSPMM_FORCE_BN": "192"}, {"NMSPMM_FORCE_SPLITK": "3"},
    {"NMSPMM_FORCE_XS": "1"}, {"NMSPMM_FORCE_PAIR": "1"}, {"NMSPMM_FORCE_PAIR": "1", "NMSPMM_FORCE_BN": "224"},
    {"NMSPMM_FORCE_GRID": "5"}], ids=lambda d: ",".join(f"{k[13:]}={v}" for k, v in d.items()))
@pytest.mark.parametrize("out", ["int8", "bfloat16"])
def test_every_kernel_variant_runs_the_output_stage(monkeypatch, plan, out):
    W, X, s, b, acc = _int8_problem(2, 4)
    for k, v in plan.items():
        monkeypatch.setenv(k, v)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Y = nm.nm_spmm_ex(h, X.cuda(), scale=s.cuda(), bias=b.cuda(), out=out, out_scale=0.25)
    torch.cuda.synchronize()
    ref = oracle.epilogue(acc, s.numpy(), b.numpy(), "none", out, 0.25)
    assert np.array_equal(_gpu_np(Y), ref["exact"])


def test_k3072_pair_kernel_int8_requant():
    # fc2-like: 4 KB of X per token selects the CTA-pair kernel
    W, X, s, b, acc = _int8_problem(2, 4, T=260, K=3072, n_out=384, seed=41)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Y = nm.nm_spmm_ex(h, X.cuda(), scale=s.cuda(), bias=b.cuda(), out="int8", out_scale=0.125)
    torch.cuda.synchronize()
    ref = oracle.epilogue(acc, s.numpy(), b.numpy(), "none", "int8", 0.125)
    assert np.array_equal(Y.cpu().numpy(), ref["exact"])


def test_fixed_stages_are_the_same_values():
    W, X, s, b, acc = _int8_problem(2, 4)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Xd, sd = X.cuda(), s.cuda()
    a = nm.nm_spmm(h, Xd, scale=sd)
    c = nm.nm_spmm_ex(h, Xd, scale=sd, out="float32")
    assert torch.equal(a, c)
    assert torch.equal(nm.nm_spmm(h, Xd), nm.nm_spmm_ex(h, Xd))
    # (float)acc without a scale goes through the runtime stage: same values as int32 -> fp32
    f = nm.nm_spmm_ex(h, Xd, out="float32")
    assert torch.equal(f, nm.nm_spmm(h, Xd).float())


def test_full_size_fc1_int8_gelu_sampled():
    l = next(x for x in inputs.vit_b_int8(patterns=("2:4",)) if x.name == "vitb.fc1")
    W, X, s = l.weight(), l.activation(), l.scale()
    b = inputs.normal_f32((l.n_out,), 5.0, 77)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Y = nm.nm_spmm_ex(h, X.cuda(), scale=s.cuda(), bias=b.cuda(), act="gelu", out="int8", out_scale=0.5)
    torch.cuda.synchronize()
    rows = np.r_[0:40, 6000:6040, l.T - 50:l.T]
    vals, idx = oracle.compress(W.numpy(), 2, 4)
    Wm = oracle.decompress(vals, idx, l.n_out, l.K, 2, 4)
    acc = oracle.gemm(np.ascontiguousarray(X.numpy()[rows]), Wm)
    r = oracle.epilogue(acc, s.numpy(), b.numpy(), "gelu", "int8", 0.5)
    q = Y.cpu().numpy()[rows].astype(np.int64)
    diff = np.abs(q - r["q"].astype(np.int64))
    assert diff.max() <= 1 and (diff == 0).mean() > 0.999


def test_ragged_and_empty():
    W, X, s, b, acc = _int8_problem(2, 4)
    h = nm.nm_compress(W.cuda(), 2, 4)
    for T in (1, 17, 129):
        Y = nm.nm_spmm_ex(h, X[:T].contiguous().cuda(), scale=s.cuda(), bias=b.cuda(), out="int8", out_scale=0.25)
        torch.cuda.synchronize()
        ref = oracle.epilogue(acc[:T], s.numpy(), b.numpy(), "none", "int8", 0.25)
        assert np.array_equal(Y.cpu().numpy(), ref["exact"])
    Y0 = nm.nm_spmm_ex(h, X[:0].contiguous().cuda(), bias=b.cuda(), out="int8")
    assert Y0.shape == (0, N0)


def _raw_ex(h, X, Y, out, act, scale=None, bias=None, out_scale=1.0):
    ep = nm.NMEpilogue(out, act, None if scale is None else scale.data_ptr(),
                       None if bias is None else bias.data_ptr(), out_scale)
    return nm.lib().nm_spmm_ex(h.raw, X.data_ptr(), X.shape[0], Y.data_ptr(), ctypes.byref(ep), None)


def test_rejected_combinations():
    W, X, s, b, acc = _int8_problem(2, 4)
    h = nm.nm_compress(W.cuda(), 2, 4)
    Xd = X.cuda()
    Y = torch.empty((T0, N0), dtype=torch.int32, device="cuda")
    bd = b.cuda()
    assert _raw_ex(h, Xd, Y, 1, 0, bias=bd) == nm.NM_ERR_INVALID              # int32 with a bias
    assert _raw_ex(h, Xd, Y, 1, 1) == nm.NM_ERR_INVALID                       # int32 with GELU
    assert _raw_ex(h, Xd, Y, 5, 0, out_scale=0.0) == nm.NM_ERR_INVALID        # int8, out_scale 0
    assert _raw_ex(h, Xd, Y, 5, 0, out_scale=float("inf")) == nm.NM_ERR_INVALID
    assert _raw_ex(h, Xd, Y, 9, 0) == nm.NM_ERR_INVALID                       # unknown output type
    assert _raw_ex(h, Xd, Y, 2, 7) == nm.NM_ERR_INVALID                       # unknown activation
    Wf = inputs.float_normal((N0, K0), 0.02, 5, inputs.FP16)
    hf = nm.nm_compress(Wf.cuda(), 2, 4)
    Xf = inputs.float_normal((T0, K0), 1.0, 6, inputs.FP16).cuda()
    assert _raw_ex(hf, Xf, Y, 5, 0) == nm.NM_ERR_UNSUPPORTED                  # int8 out, fp16 in
    assert _raw_ex(hf, Xf, Y, 1, 0) == nm.NM_ERR_UNSUPPORTED                  # int32 out, fp16 in
    torch.cuda.synchronize()
