"""Host logic of the calibrated LUT latency predictor (no GPU)."""
import numpy as np
import pytest

from structured_sparse_gemm_compress_b200 import lut


def _table():
    # latency linear in T per (shape, pattern): us = c0 + c1 * T
    coef = {("2:4", 768, 2304): (5.0, 0.002), ("dense", 768, 2304): (6.0, 0.003),
            ("2:4", 3072, 768): (4.0, 0.0015), ("dense", 3072, 768): (5.0, 0.0025)}
    t = {}
    for (p, K, n), (c0, c1) in coef.items():
        for T in (197, 1000, 50432):
            t[(K, n, p, T)] = c0 + c1 * T
    return lut.LatencyLUT(t), coef


def test_lookup_exact_interpolated_and_extrapolated():
    L, coef = _table()
    c0, c1 = coef[("2:4", 768, 2304)]
    assert L.lookup(768, 2304, "2:4", 1000) == pytest.approx(c0 + c1 * 1000)
    # between grid points the table is linear in T, so a linear law is reproduced
    for T in (500, 12608, 30000):
        assert L.lookup(768, 2304, "2:4", T) == pytest.approx(c0 + c1 * T, rel=1e-12)
    # outside the grid: the nearest pair extrapolates the same line
    for T in (1, 100000):
        assert L.lookup(768, 2304, "2:4", T) == pytest.approx(c0 + c1 * T, rel=1e-12)
    with pytest.raises(KeyError):
        L.lookup(768, 2304, "1:4", 1000)


def test_interpolation_uses_the_bracketing_pair():
    t = {(8, 8, "2:4", 10): 1.0, (8, 8, "2:4", 20): 3.0, (8, 8, "2:4", 40): 4.0}
    L = lut.LatencyLUT(t)
    assert L.lookup(8, 8, "2:4", 15) == pytest.approx(2.0)
    assert L.lookup(8, 8, "2:4", 30) == pytest.approx(3.5)
    assert L.lookup(8, 8, "2:4", 50) == pytest.approx(4.5)
    assert L.lookup(8, 8, "2:4", 5) == pytest.approx(0.0)


def test_calibration_recovers_a_linear_law():
    L, _ = _table()
    layers = [lut.LayerSpec("qkv", 768, 2304), lut.LayerSpec("fc2", 3072, 768)]
    samples = []
    for i, T in enumerate((197, 1000, 5000, 20000, 50432)):
        for n_layers in (2, 4, 6):
            ls = (layers * 3)[:n_layers]
            asg = lut.random_assignment(n_layers, seed=10 * i + n_layers, patterns=("2:4", "dense"))
            samples.append((ls, asg, T, 1.1 * L.raw_sum(ls, asg, T) + 2.5 * n_layers))
    a, b = L.calibrate(samples)
    assert a == pytest.approx(1.1, rel=1e-9) and b == pytest.approx(2.5, rel=1e-9)
    ls, asg = layers * 2, ["2:4", "dense", "dense", "2:4"]
    assert L.predict(ls, asg, 777) == pytest.approx(1.1 * L.raw_sum(ls, asg, 777) + 2.5 * 4)


def test_calibration_with_one_sample_scales_only():
    L, _ = _table()
    ls = [lut.LayerSpec("qkv", 768, 2304)]
    a, b = L.calibrate([(ls, ["2:4"], 1000, 2 * L.raw_sum(ls, ["2:4"], 1000))])
    assert (a, b) == (pytest.approx(2.0), 0.0)


def test_json_round_trip_and_argument_checks():
    L, _ = _table()
    L.a, L.b = 1.25, 0.5
    L2 = lut.LatencyLUT.from_json(L.to_json())
    assert L2.table == L.table and (L2.a, L2.b) == (1.25, 0.5)
    with pytest.raises(ValueError):
        L.raw_sum([lut.LayerSpec("x", 768, 2304)], ["2:4", "2:4"], 197)


def test_vit_b_layers_and_assignments():
    ls = lut.vit_b_layers()
    assert len(ls) == 48 and ls[2] == lut.LayerSpec("b0.fc1", 768, 3072)
    a1, a2 = lut.random_assignment(48, 5), lut.random_assignment(48, 5)
    assert a1 == a2 and set(a1) <= set(lut.PATTERNS)


def test_pattern_names_cover_both_families():
    assert lut.pattern_nm("2:4") == (2, 4, False)
    assert lut.pattern_nm("dense") == (4, 4, False)
    assert lut.pattern_nm("t2:8") == (2, 8, True)
    assert lut.pattern_nm("t4:8") == (4, 8, True)
    with pytest.raises(KeyError):
        lut.pattern_nm("t3:8")
    asg = lut.random_assignment(200, 3, tuple(lut.PATTERNS) + tuple(lut.TILE_PATTERNS))
    assert set(asg) == set(lut.PATTERNS) | set(lut.TILE_PATTERNS)


def test_calibration_recovers_a_per_family_term():
    """measured = 1.1 * sum + 0.5 per layer + 3.0 per tile-shared layer is recovered
    exactly, and predict() applies all three terms."""
    layers = lut.vit_b_layers(blocks=1)
    table = {(l.K, l.n_out, p, 100): 10.0 + i + 3 * j for i, l in enumerate(layers)
             for j, p in enumerate(("2:4", "t2:8", "dense"))}
    L = lut.LatencyLUT(table)
    rng = np.random.default_rng(0)
    samples = []
    for _ in range(8):
        asg = [rng.choice(["2:4", "t2:8", "dense"]) for _ in layers]
        meas = 1.1 * L.raw_sum(layers, asg, 100) + 0.5 * len(layers) + 3.0 * lut.n_tile_layers(asg)
        samples.append((layers, asg, 100, meas))
    L.calibrate(samples)
    assert (L.a, L.b, L.c) == pytest.approx((1.1, 0.5, 3.0))
    asg = ["t2:8", "2:4", "t2:8", "dense"]
    assert L.predict(layers, asg, 100) == pytest.approx(1.1 * L.raw_sum(layers, asg, 100) + 2.0 + 6.0)
    L2 = lut.LatencyLUT.from_json(L.to_json())
    assert L2.c == pytest.approx(3.0)


def test_stratified_assignments_set_the_tile_share():
    asgs = lut.stratified_assignments(48, 7)
    assert [lut.n_tile_layers(a) for a in asgs] == [0, 12, 24, 36, 48]
    for a in asgs:
        assert len(a) == 48 and set(a) <= set(lut.PATTERNS) | set(lut.TILE_PATTERNS)
    assert lut.stratified_assignments(48, 7) == asgs                  # seeded
