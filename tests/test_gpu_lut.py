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
    for T in Ts:
        for i in range(3):
            asg = lut.random_assignment(len(layers), 50 + i)
            meas = lut.measure_sequence(layers, asg, T, reps=3, ws=ws)
            pred = L.predict(layers, asg, T)
            assert abs(pred - meas) <= 0.2 * meas, (T, asg, pred, meas)
    # the profiled table answers any T through interpolation
    assert L.lookup(768, 2304, "2:4", 2000) > 0
