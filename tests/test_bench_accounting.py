"""bench.py's accounting on CPU: algorithmic bytes, the roofline point and the
whole-job throughput, checked against numbers worked out by hand from the
layer shapes (ViT-B at T = 12608); and the clock sampler's placement of its
NVML readings around the timed region (against a stand-in for pynvml)."""
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


class _FakeNvml:
    """Stands in for pynvml: records whether each power reading happened inside
    the sampler's timed region."""
    NVML_CLOCK_SM = 1

    def __init__(self):
        self.sampler = None
        self.power_inside = []
        self.clock_reads = 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        return "gpu0"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.clock_reads += 1
        return 1965 if self.clock_reads % 2 else 1800

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4  # sw_power_cap

    def nvmlDeviceGetPowerUsage(self, h):
        self.power_inside.append(bool(self.sampler and self.sampler._inside))
        return 400_000  # mW


def test_clock_sampler_reads_power_only_outside_the_timed_region(monkeypatch):
    """Power readings through NVML while the GPU ran the step stretched the timed
    region, so the sampler polls clocks and reasons inside it and reads the
    power just before and just after."""
    import sys
    import time
    import types

    import bench

    fake = _FakeNvml()
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x1b, pci_device_id=0)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda dev: props)
    with bench.NvmlSampler(0) as s:
        fake.sampler = s
        s.mark_start()
        time.sleep(0.03)
        s.poke()
        s.mark_end()
    summary = s.summary()
    assert fake.power_inside == [False, False]  # one reading before, one after the region
    assert summary["samples_in_timed_region"] >= 2 and fake.clock_reads >= 2
    assert summary["reasons"] == ["sw_power_cap"]
    assert summary["sm_max_mhz"] == 1965 and summary["sm_min_mhz"] in (1800, 1965)
    assert summary["power_w_max"] == 400.0
