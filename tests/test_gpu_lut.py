"""The calibrated LUT latency predictor on the GPU: profiled table + calibration
predict held-out layer-wise sequences close to their measured latency."""
import pytest

from structured_sparse_gemm_compress_b200 import lut

pytestmark = pytest.mark.gpu


def test_lut_predicts_held_out_sequences():
    layers = lut.vit_b_layers(blocks=2)
    shapes = sorted({(l.K, l.n_out) for l in layers})
    Ts = [197, 4096]
    ws = lut._Workspace()
    L = lut.profile(shapes, list(lut.PATTERNS), Ts, reps=10, ws=ws)
    assert len(L.table) == len(shapes) * len(lut.PATTERNS) * len(Ts)
    assert all(us > 0 for us in L.table.values())
    calib = [(layers, lut.random_assignment(len(layers), 10 + i), T,
              lut.measure_sequence(layers, lut.random_assignment(len(layers), 10 + i), T, reps=3, ws=ws))
             for T in Ts for i in range(3)]
    L.calibrate(calib)
    errs = []
    for T in Ts:
        for i in range(3):
            asg = lut.random_assignment(len(layers), 50 + i)
            meas = lut.measure_sequence(layers, asg, T, reps=3, ws=ws)
            pred = L.predict(layers, asg, T)
            errs.append(abs(pred - meas) / meas)
            # a latency budget enforced through the predictor is only as good as this bound
            assert errs[-1] <= 0.10, (T, asg, pred, meas)
    print("held-out relative errors:", [round(e, 4) for e in errs])
    assert sum(errs) / len(errs) <= 0.05, errs
    # the profiled table answers any T through interpolation
    assert L.lookup(768, 2304, "2:4", 2000) > 0


def test_lut_with_tile_shared_patterns():
    """Tile-shared patterns are profiled on the gather kernel and sequences
    that mix both families are predicted like the others."""
    layers = lut.vit_b_layers(blocks=1)
    shapes = sorted({(l.K, l.n_out) for l in layers})
    pats = ["2:4", "dense", "t2:8", "t4:8"]
    ws = lut._Workspace()
    L = lut.profile(shapes, pats, [2048], reps=10, ws=ws)
    assert all(us > 0 for us in L.table.values())
    calib = []
    for i in range(3):
        asg = lut.random_assignment(len(layers), 70 + i, tuple(pats))
        calib.append((layers, asg, 2048, lut.measure_sequence(layers, asg, 2048, reps=3, ws=ws)))
    L.calibrate(calib)
    for i in range(3):
        asg = lut.random_assignment(len(layers), 90 + i, tuple(pats))
        meas = lut.measure_sequence(layers, asg, 2048, reps=3, ws=ws)
        assert abs(L.predict(layers, asg, 2048) - meas) <= 0.10 * meas, (asg, meas)


def test_tile_shared_keeps_at_most_the_per_row_mass():
    """A shared pattern per 128 rows cannot keep more |w| than each row's own best."""
    import torch

    from structured_sparse_gemm_compress_b200 import inputs, search
    W = inputs.int8_uniform((384, 768), -127, 127, 5).cuda()
    for N, M in ((2, 8), (4, 8), (1, 4)):
        assert search.kept_mass(W, N, M, tile=True) <= search.kept_mass(W, N, M) + 1e-6
    assert search.kept_mass(W, 4, 4, tile=True) == float(W.to(torch.float64).abs().sum())
