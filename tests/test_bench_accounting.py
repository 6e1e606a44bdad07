"""bench.py's accounting on CPU: algorithmic bytes, the roofline point and the
whole-job throughput, checked against numbers worked out by hand from the
layer shapes (ViT-B at T = 12608)."""
import pytest

import bench
from structured_sparse_gemm_compress_b200 import inputs

PK = {"hbm_gbs": 6553.0, "bf16_tflops": 1654.0}


def _layer(name, nm):
    return next(l for l in inputs.vit_b_int8() if l.name == name and l.nm == nm)


def test_alg_bytes_qkv_2of4_by_hand():
    l = _layer("vitb.qkv", "2:4")
    T, K, n = 12608, 768, 2304
    kept = n * (K // 4) * 2                       # 884,736 kept int8 values
    want = T * K + kept + kept * 2 // 8 + T * n * 4 + 4 * n   # X + values + 2-bit positions + fp32 Y + scale
    assert bench.alg_bytes(l) == want
    assert bench.alg_bytes_any(l) == want
    assert 126e6 < want < 128e6                   # ~127 MB


def test_alg_bytes_dense_and_narrow_outputs():
    l = _layer("vitb.fc2", "4:8")
    T, K, n = 12608, 3072, 768
    kept = n * (K // 8) * 4
    assert bench.alg_bytes(l) == T * K + kept + kept * 3 // 8 + T * n * 4 + 4 * n
    # int8 output with a bias: 1 byte per output element, 4 bytes of bias per channel
    assert bench.alg_bytes_any(l, out_es=1, biased=True) == T * K + kept + kept * 3 // 8 + T * n + 8 * n


def test_roofline_point_hbm_bound():
    l = _layer("vitb.fc1", "2:4")
    us = 40.0
    rp = bench.roofline_point(l, us, PK)
    ops = 2 * 12608 * 768 * 3072
    t_hbm = bench.alg_bytes(l) / (PK["hbm_gbs"] * 1e9) * 1e6
    t_tc = ops / (PK["bf16_tflops"] * 2 * 2 * 1e12) * 1e6     # INT8 = 2 x bf16, 2:4 sparse = 2 x dense
    assert t_hbm > t_tc
    assert rp["bound"] == "hbm"
    assert rp["roofline_us"] == pytest.approx(t_hbm, abs=0.01)
    assert rp["frac"] == pytest.approx(t_hbm / us, abs=1e-3)
    assert rp["dense_eq_tops"] == pytest.approx(ops / us / 1e6, abs=0.1)


def test_roofline_point_gather_uses_kept_work_on_the_dense_pipe():
    l = _layer("vitb.fc2", "2:8")
    ops = 2 * 12608 * 3072 * 768
    rp_sparse = bench.roofline_point(l, 1000.0, PK)
    rp_gather = bench.roofline_point(l, 1000.0, PK, gather=True)
    # both far below the time: HBM decides either way; the tensor time differs
    t_tc_sparse = ops / (PK["bf16_tflops"] * 2 * 2 * 1e12) * 1e6
    t_tc_gather = ops * 2 / 8 / (PK["bf16_tflops"] * 2 * 1e12) * 1e6
    assert t_tc_gather == pytest.approx(t_tc_sparse / 2)
    assert rp_sparse["roofline_us"] == rp_gather["roofline_us"]


def test_whole_job_tops():
    # 4 steps of 1e12 dense-equivalent ops on 2 ranks in 10 ms: 800 TOPS
    assert bench.whole_job_tops(10**12, 4, 2, 10.0) == pytest.approx(800.0)
