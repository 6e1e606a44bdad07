#!/usr/bin/env python
"""Benchmark of the N:M sparse GEMM path on B200.

One step = the whole path over the ViT-B/16 INT8 linear-layer set at batch 64
(T = 12608 tokens; QKV 768->2304, proj 768->768, FC1 768->3072, FC2 3072->768;
N:M in {1:4, 2:4, 2:8, 4:8}; per-output-channel fp32 scale, fp32 Y):
for each of the 16 (layer, N:M) problems, re-pack the layer's weight
(nm_recompress: top-N select + packed operand image) and run nm_spmm.
Inputs are seeded synthetic tensors with the workload's shapes and value
distributions (structured_sparse_gemm_compress_b200.inputs); every step
streams about 1.7 GB, far more than the 126 MB L2, so no repeat is L2-warm.

Metric: dense-equivalent TOPS = sum(2*T*K*n_out) / time, whole job (all ranks).
Multi-GPU: replicas only -- tokens are independent, each rank runs its own
batch on its own GPU with no data-path collective (weak scaling); the barrier
and the max-over-ranks timing use torch.distributed.

`--impl reference` times the CPU oracle (the only reference implementation
there is) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from structured_sparse_gemm_compress_b200 import inputs  # noqa: E402

METRIC = "N:M SpMM effective TOPS (dense-equiv) on ViT-B layers; % of sparse-TC roofline"
UNIT = "TOPS"
WORKLOAD = "ViT-B/16 INT8 linear set, batch 64 (T=12608), N:M in {1:4,2:4,2:8,4:8}, per-channel fp32 scale"
CPU_SAMPLE_ROWS = 9216      # ~10 s of oracle work on a 16-thread host (1536 rows took 1.7 s there)
REF_SAMPLE_ROWS = 192       # per reference-arm step, so --steps 20 stays within a few minutes


_ONLY: list[str] = []


def layers():
    """The 16 (layer, N:M) problems, or the subset named by --only (name/N:M)."""
    ls = inputs.vit_b_int8()
    if _ONLY:
        ls = [l for l in ls if f"{l.name}/{l.nm}" in _ONLY]
        if not ls:
            raise SystemExit(f"--only matched no problem: {_ONLY}")
    return ls


def alg_bytes(l) -> int:
    """Algorithmic bytes of one SpMM launch: X + packed W (kept values + log2(M)
    bits of position each) + Y + scale."""
    import math
    kept = l.n_out * (l.K // l.M) * l.N
    wbytes = kept + (kept * math.ceil(math.log2(l.M)) + 7) // 8 if l.N != l.M else l.n_out * l.K
    ybytes = l.T * l.n_out * 4
    return l.T * l.K + wbytes + ybytes + (4 * l.n_out if l.scaled else 0)


def pack_bytes(l) -> int:
    """Algorithmic bytes of one re-pack: read W, write canonical values + positions."""
    kept = l.n_out * (l.K // l.M) * l.N
    return l.n_out * l.K + kept + (kept + 1) // 2


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while running;
    the summary keeps the samples taken inside the window marked by
    ``mark_start``/``mark_end`` (the timed region)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def poke(self):
        pass

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        import datetime

        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        inside = []
        if self.t0 is not None and self.t1 is not None:
            for r in rows:
                try:
                    ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    continue
                if self.t0 <= ts <= self.t1:
                    inside.append(r)
        window = len(inside)
        rows = [r[1:] for r in (inside or rows)]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        busy = [s for s in sm if s > 0.5 * max(mx or [1])] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "samples_in_timed_region": window}


class NvmlSampler:
    """SM clock, its maximum and the clock-event reasons of the GPU this
    process uses (found by PCI bus id), polled by NVML from a thread about
    every half millisecond between ``mark_start`` and ``mark_end``, so even a
    timed region of a few milliseconds is covered.  The power draw is read only
    just before and just after the region: on B200 an NVML power reading taken
    while the GPU was busy stretched a 20-step region up to 7x (clock and reason
    readings did not).  Falls back to ``ClockSampler`` (nvidia-smi every 50 ms)
    when NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.power = []
        self._run = False
        self._thread = None
        self._nvml = None
        self._h = None
        self._fallback = None
        self._inside = False

    def __enter__(self):
        import threading
        try:
            import pynvml

            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(self.dev)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
            self._fallback = ClockSampler(self.dev).__enter__()
            return self
        self._run = True
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()
        return self

    def _sample(self):
        n = self._nvml
        get_reasons = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            n.nvmlDeviceGetCurrentClocksThrottleReasons
        try:
            sm = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
            rs = get_reasons(self._h)
            self.samples.append((sm, rs, None))
        except Exception:
            pass

    def _power(self):
        try:
            self.power.append(self._nvml.nvmlDeviceGetPowerUsage(self._h) / 1000.0)
        except Exception:
            pass

    def _poll(self):
        while self._run:
            if self._inside:
                self._sample()
                time.sleep(0.0005)
            else:
                time.sleep(0.0002)

    def poke(self):
        """One sample taken now (call while the GPU is busy inside the region)."""
        if self._nvml is not None and self._inside:
            self._sample()

    def mark_start(self):
        if self._fallback is not None:
            return self._fallback.mark_start()
        self._power()
        self._inside = True

    def mark_end(self):
        if self._fallback is not None:
            return self._fallback.mark_end()
        self._inside = False
        self._power()



    def __exit__(self, *exc):
        if self._fallback is not None:
            return self._fallback.__exit__(*exc)
        self._run = False
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self) -> dict:
        if self._fallback is not None:
            return self._fallback.summary()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": ["unsampled"],
                    "samples": 0, "samples_in_timed_region": 0, "source": "nvml"}
        sm = [x[0] for x in self.samples]
        reasons = sorted({name for _, rs, _ in self.samples for name, bit in self.REASONS if rs & bit})
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "power_w_max": round(max(self.power), 1) if self.power else None,
                "power_read": "just before and just after the timed region",
                "samples": len(sm), "samples_in_timed_region": len(sm),
                "source": "nvml clocks and reasons, ~0.5 ms polling"}


# --------------------------------------------------------------------------- multi-rank plumbing


def rank_env() -> tuple[int, int, int]:
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time: replicas finish together only when the slowest does."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(ops_per_rank_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank processes its own batch (weak scaling)."""
    return ops_per_rank_step * steps * world / (ms * 1e-3) / 1e12


# --------------------------------------------------------------------------- reference arm (CPU oracle)


def cpu_oracle_run(ls, rows: int):
    """Oracle over a sample: the first `rows` tokens of every problem (compress,
    decompress, triple-loop GEMM).  Returns (seconds, dense-equivalent ops)."""
    import oracle

    data = []
    for l in ls:
        W = l.weight().numpy()
        X = l.activation(T=rows).numpy()
        s = l.scale().numpy()
        data.append((l, W, X, s))
    t0 = time.perf_counter()
    ops = 0
    for l, W, X, s in data:
        oracle.spmm(X, W, l.N, l.M, scale=s)
        ops += 2 * rows * l.K * l.n_out
    return time.perf_counter() - t0, ops


def run_reference(args, rank: int) -> None:
    if rank != 0:
        return
    import oracle

    oracle.build()
    ls = layers()
    for _ in range(args.warmup):
        cpu_oracle_run(ls, 16)
    secs, ops = 0.0, 0
    rows = args.cpu_rows or REF_SAMPLE_ROWS
    for _ in range(args.steps):
        s, o = cpu_oracle_run(ls, rows)
        secs += s
        ops += o
    value = ops / secs / 1e12
    sample = (f"first {rows} of 12608 tokens of each of the 16 (layer, N:M) problems per step "
              f"(compress + decompress + triple-loop GEMM), {args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
        "data": "synthetic", "config": {"workload": WORKLOAD + " (CPU oracle on a token sample)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- other workloads


def roofline_point(l, us: float, pk: dict, out_es: int | None = None, biased: bool = False,
                   gather: bool = False) -> dict:
    """Roofline of one problem: t = max(ops / tensor peak, bytes / HBM peak).

    Tensor peaks: INT8 dense = the INT8 peak measured in the same run
    (``pk["int8_tops"]``; 2 x the measured bf16 peak, NVIDIA's nominal ratio,
    when absent), FP16/BF16 dense = the measured bf16 peak, 2:4-sparse = 2 x
    dense (1:4, 2:4, 2:8 run on the sparse pipe; 4:8 and N = M on the dense
    pipe).
    gather: tile-shared patterns, whose MMAs run on the dense pipe over the kept
    k only (N/M of the dense-equivalent work)."""
    if l.dtype == inputs.INT8:
        dense_peak = pk.get("int8_tops") or pk["bf16_tflops"] * 2.0
    else:
        dense_peak = pk["bf16_tflops"]
    sparse = (l.N, l.M) in ((1, 4), (2, 4), (2, 8))
    tc_peak = dense_peak * (2.0 if sparse else 1.0)
    ops = l.dense_ops()
    t_tc = ops / (tc_peak * 1e12) * 1e6
    if gather:
        t_tc = ops * l.N / l.M / (dense_peak * 1e12) * 1e6
    bytes_ = alg_bytes_any(l, out_es, biased)
    t_hbm = bytes_ / (pk["hbm_gbs"] * 1e9) * 1e6
    t_roof = max(t_tc, t_hbm)
    return {"us": round(us, 2), "dense_eq_tops": round(ops / us / 1e6, 1),
            "useful_tops": round(l.kept_ops() / us / 1e6, 1),
            "bound": "tensor" if t_tc > t_hbm else "hbm", "roofline_us": round(t_roof, 2),
            "frac": round(t_roof / us, 3)}


def alg_bytes_any(l, out_es: int | None = None, biased: bool = False) -> int:
    """Algorithmic bytes of one SpMM launch for any dtype/output (out_es: bytes
    per output element when not the default of the dtype)."""
    import math
    es = 1 if l.dtype == inputs.INT8 else 2
    kept = l.n_out * (l.K // l.M) * l.N
    wbytes = (kept * es + (kept * math.ceil(math.log2(l.M)) + 7) // 8) if l.N != l.M else l.n_out * l.K * es
    if out_es is None:
        out_es = 4 if l.dtype == inputs.INT8 else 2
    return (l.T * l.K * es + wbytes + l.T * l.n_out * out_es + (4 * l.n_out if l.scaled else 0)
            + (4 * l.n_out if biased else 0))


def run_lut(args) -> None:
    """Calibrated LUT latency predictor on the 48 ViT-B linears: profile every
    (shape, pattern) at T = 197 and 50432, calibrate on random layer-wise
    assignments, then report the prediction error on held-out assignments and
    on the mixed sequence (seed 5), each against its measured latency."""
    from structured_sparse_gemm_compress_b200 import lut

    torch.cuda.set_device(0)
    layers = lut.vit_b_layers()
    shapes = sorted({(l.K, l.n_out) for l in layers})
    Ts = [197, 50432]
    ws = lut._Workspace()
    t0 = time.time()
    L = lut.profile(shapes, list(lut.PATTERNS), Ts, reps=20, ws=ws)
    t_prof = time.time() - t0
    calib = []
    for T in Ts:
        for i in range(4):
            asg = lut.random_assignment(len(layers), 100 + i)
            calib.append((layers, asg, T, lut.measure_sequence(layers, asg, T, reps=3, ws=ws)))
    L.calibrate(calib)
    mixed = [("dense" if l.N == l.M else l.nm) for l in inputs.vit_b_mixed(197)]
    per_t, errs = {}, []
    for T in Ts:
        rows = []
        for i, asg in enumerate([lut.random_assignment(len(layers), 200 + i) for i in range(6)] + [mixed]):
            meas = lut.measure_sequence(layers, asg, T, reps=3, ws=ws)
            pred = L.predict(layers, asg, T)
            rows.append({"assignment": "mixed seed 5" if i == 6 else f"random seed {200 + i}",
                         "measured_us": round(meas, 1), "predicted_us": round(pred, 1),
                         "raw_lut_sum_us": round(L.raw_sum(layers, asg, T), 1),
                         "err_pct": round(100 * (pred - meas) / meas, 2)})
            errs.append(abs(pred - meas) / meas)
        per_t[str(T)] = rows
    line = {"config": {"workload": "calibrated LUT latency predictor, 48 ViT-B linears, INT8 + scale, "
                                   "patterns {dense,4:8,2:4,2:8,1:4}, T in {197, 50432}"},
            "metric": "mean |predicted - measured| / measured over held-out layer-wise assignments",
            "value": round(100 * float(np.mean(errs)), 3), "unit": "%", "higher_is_better": False,
            "max_err_pct": round(100 * float(np.max(errs)), 3),
            "calibration": {"a": round(L.a, 4), "b_us_per_layer": round(L.b, 3), "samples": len(calib)},
            "lut_entries": len(L.table), "profile_s": round(t_prof, 1), "per_T": per_t,
            "data": "synthetic", "dtype": "int8"}
    print(json.dumps(line), flush=True)


def run_search(args) -> None:
    """Latency-constrained layer-wise N:M search over the 48 ViT-B linears at
    T = 50432 with the calibrated LUT: the evolutionary solver against the
    exact (dynamic-programming) optimum and the greedy repair, proxy quality =
    kept |w| fraction of the seeded weights, the chosen configuration measured."""
    from structured_sparse_gemm_compress_b200 import lut, search

    torch.cuda.set_device(0)
    layers = lut.vit_b_layers()
    T = 50432
    shapes = sorted({(l.K, l.n_out) for l in layers})
    ws = lut._Workspace()
    L = lut.profile(shapes, list(lut.PATTERNS), [T], reps=10, ws=ws)
    calib = []
    for i in range(4):
        asg = lut.random_assignment(len(layers), 300 + i)
        calib.append((layers, asg, T, lut.measure_sequence(layers, asg, T, reps=3, ws=ws)))
    L.calibrate(calib)
    keep, total = {}, {}
    for i, l in enumerate(layers):
        W = inputs.int8_uniform((l.n_out, l.K), -127, 127, 7000 + i).cuda()
        total[l.name] = float(W.to(torch.float64).abs().sum())
        for p, (N, M) in lut.PATTERNS.items():
            keep[(l.name, p)] = search.kept_mass(W, N, M)
    pats = list(lut.PATTERNS)
    dense = L.predict(layers, ["dense"] * len(layers), T)
    probe = search.make_problem(layers, L, T, keep, total, 1e12, pats)
    fastest = probe.latency(np.argmin(probe.lat, axis=1))
    rows = []
    for frac in (0.25, 0.5, 0.75):
        budget = dense - frac * (dense - fastest)
        prob = search.make_problem(layers, L, T, keep, total, budget, pats)
        t0 = time.time()
        ga = search.solve_evolutionary(prob, pop=64, generations=150, seed=1)
        t_ga = time.time() - t0
        ex = search.solve_exact(prob, resolution_us=0.05)
        gr = search.solve_greedy(prob)
        asg = [pats[i] for i in ga]
        meas = lut.measure_sequence(layers, asg, T, reps=3, ws=ws)
        rows.append({"budget_us": round(budget, 1), "budget_cut_of_dense_to_fastest": frac,
                     "ga_quality": round(prob.quality(ga), 6), "exact_quality": round(prob.quality(ex), 6),
                     "greedy_quality": round(prob.quality(gr), 6), "ga_s": round(t_ga, 2),
                     "ga_predicted_us": round(prob.latency(ga), 1), "ga_measured_us": round(meas, 1),
                     "measured_over_budget_pct": round(100 * (meas - budget) / budget, 2),
                     "pattern_counts": {p: asg.count(p) for p in pats}})
    gap = max(r["exact_quality"] - r["ga_quality"] for r in rows)
    line = {"config": {"workload": "latency-constrained layer-wise N:M search, 48 ViT-B linears, T=50432, "
                                   "calibrated LUT, proxy quality = kept |w| fraction (seeded INT8 weights)"},
            "metric": "largest quality gap of the evolutionary solver to the exact optimum over three budgets",
            "value": round(gap, 6), "unit": "fraction of total |w|", "higher_is_better": False,
            "all_dense_predicted_us": round(dense, 1), "all_fastest_predicted_us": round(fastest, 1),
            "calibration": {"a": round(L.a, 4), "b_us_per_layer": round(L.b, 3)}, "budgets": rows,
            "data": "synthetic", "dtype": "int8"}
    print(json.dumps(line), flush=True)


def run_cosearch(args) -> None:
    """Search-kernel co-design on the 48 ViT-B linears at T = 12608: the
    layer-wise search over per-row N:M patterns alone, and over those plus
    tile-shared patterns run through the activation-gather kernel, with one
    calibrated LUT profiled on the real kernels.  Reports the fastest
    configuration of each family (measured), and per latency budget (across the
    per-row range and below its minimum) the exact optimum of both searches
    (quality = kept |w| fraction), the evolutionary solver on the joint one and
    its configuration measured."""
    from structured_sparse_gemm_compress_b200 import lut, search

    torch.cuda.set_device(0)
    layers = lut.vit_b_layers()
    T = 12608
    shapes = sorted({(l.K, l.n_out) for l in layers})
    pats_ew = list(lut.PATTERNS)
    pats_all = pats_ew + list(lut.TILE_PATTERNS)
    ws = lut._Workspace()
    L = lut.profile(shapes, pats_all, [T], reps=10, ws=ws)
    calib = []
    for asg in lut.stratified_assignments(len(layers), 400) + lut.stratified_assignments(len(layers), 401):
        calib.append((layers, asg, T, lut.measure_sequence(layers, asg, T, reps=3, ws=ws)))
    L.calibrate(calib)
    keep, total = {}, {}
    for i, l in enumerate(layers):
        W = inputs.int8_uniform((l.n_out, l.K), -127, 127, 7000 + i).cuda()
        total[l.name] = float(W.to(torch.float64).abs().sum())
        for p in pats_all:
            N, M, tile = lut.pattern_nm(p)
            keep[(l.name, p)] = search.kept_mass(W, N, M, tile)
    dense = L.predict(layers, ["dense"] * len(layers), T)
    probe_ew = search.make_problem(layers, L, T, keep, total, 1e12, pats_ew)
    probe_all = search.make_problem(layers, L, T, keep, total, 1e12, pats_all)
    fast_ew, fast_all = np.argmin(probe_ew.lat, axis=1), np.argmin(probe_all.lat, axis=1)
    fastest_ew, fastest_all = probe_ew.latency(fast_ew), probe_all.latency(fast_all)
    meas_fast_ew = lut.measure_sequence(layers, [pats_ew[i] for i in fast_ew], T, reps=3, ws=ws)
    meas_fast_all = lut.measure_sequence(layers, [pats_all[i] for i in fast_all], T, reps=3, ws=ws)
    # budgets across the per-row range, then below the per-row minimum (only the joint search reaches those)
    budgets = [dense - f * (dense - fastest_ew) for f in (0.25, 0.5, 0.75, 0.95)]
    budgets += [fastest_ew - f * (fastest_ew - fastest_all) for f in (0.5, 0.9)] if fastest_all < fastest_ew else []
    rows = []
    for budget in budgets:
        p_ew = search.make_problem(layers, L, T, keep, total, budget, pats_ew)
        p_all = search.make_problem(layers, L, T, keep, total, budget, pats_all)
        ex_ew = search.solve_exact(p_ew, resolution_us=0.01)
        ex_all = search.solve_exact(p_all, resolution_us=0.01)
        ga = search.solve_evolutionary(p_all, pop=64, generations=150, seed=1)
        asg = [pats_all[i] for i in ga]
        meas = lut.measure_sequence(layers, asg, T, reps=3, ws=ws)
        rows.append({"budget_us": round(budget, 1),
                     "exact_quality_per_row_only": round(p_ew.quality(ex_ew), 6) if ex_ew is not None else None,
                     "exact_quality_with_tile_shared": round(p_all.quality(ex_all), 6) if ex_all is not None else None,
                     "ga_quality_with_tile_shared": round(p_all.quality(ga), 6),
                     "ga_predicted_us": round(p_all.latency(ga), 1), "ga_measured_us": round(meas, 1),
                     "measured_over_budget_pct": round(100 * (meas - budget) / budget, 2),
                     "pattern_counts": {p: asg.count(p) for p in pats_all if asg.count(p)}})
    line = {"config": {"workload": "search-kernel co-design: layer-wise N:M search over 48 ViT-B linears at "
                                   "T=12608 with per-row patterns {dense,4:8,2:4,2:8,1:4} and tile-shared "
                                   "patterns {4:8,2:8,1:4} through the gather kernel (activations feature-major; "
                                   "the layout change between layers is not counted), calibrated LUT, proxy "
                                   "quality = kept |w| fraction (seeded INT8 weights)"},
            "metric": "latency of the fastest configuration, per-row patterns only against per-row plus "
                      "tile-shared gather kernels (measured sequence)",
            "value": round(100 * (meas_fast_ew - meas_fast_all) / meas_fast_ew, 2), "unit": "% lower latency",
            "higher_is_better": True,
            "fastest_per_row": {"predicted_us": round(fastest_ew, 1), "measured_us": round(meas_fast_ew, 1)},
            "fastest_joint": {"predicted_us": round(fastest_all, 1), "measured_us": round(meas_fast_all, 1),
                              "pattern_counts": {p: [pats_all[i] for i in fast_all].count(p) for p in pats_all
                                                 if [pats_all[i] for i in fast_all].count(p)}},
            "all_dense_predicted_us": round(dense, 1),
            "calibration": {"a": round(L.a, 4), "b_us_per_layer": round(L.b, 3),
                            "c_us_per_tile_shared_layer": round(L.c, 3)}, "budgets": rows,
            "lut_us_fc2": {p: round(L.lookup(3072, 768, p, T), 2) for p in pats_all},
            "data": "synthetic", "dtype": "int8"}
    print(json.dumps(line), flush=True)


def _graph_stats(launch, stream, reps: int = 20, replays: int = 11) -> tuple[float, float, float]:
    """(median, p10, p90) in us of one launch over `replays` replays of a CUDA
    graph of `reps` back-to-back launches (see _graph_us)."""
    ts = _graph_us(launch, stream, reps, replays, all_replays=True)
    q = np.percentile(ts, [50, 10, 90])
    return float(q[0]), float(q[1]), float(q[2])


def _graph_us(launch, stream, reps: int = 20, replays: int = 5, all_replays: bool = False):
    """Time (us) of one launch: `reps` launches back to back in one CUDA graph,
    events around each replay, median over `replays` replays.  Our kernels and
    cuBLAS's are timed by this same function, so launch overlap (programmatic
    dependent launch for ours, graph replay for both) and the L2 state (X and
    W resident across the repeats, Y streaming) are alike."""
    for _ in range(3):
        launch(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
        for _ in range(reps):
            launch(cap)
    g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(replays):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e3 / reps)
    del g
    return ts if all_replays else statistics.median(ts)


def measure_int8_peak(device) -> dict:
    """Dense INT8 tensor-core peak of this GPU, measured: cuBLAS int8 GEMM
    (torch._int_mm, int32 out) at 8192^3, CUDA events, best of 20.  The 2:4
    sparse INT8 peak is taken as twice this (the sparse pipe's nominal ratio)."""
    n = 8192
    a = torch.randint(-128, 128, (n, n), dtype=torch.int8, device=device)
    b = torch.randint(-128, 128, (n, n), dtype=torch.int8, device=device).t()
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(20):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return {"int8_dense_tops": 2.0 * n ** 3 / (best * 1e-3) / 1e12, "how": f"torch._int_mm {n}^3, best of 20"}


CONFIG_NAMES = ("single", "vitl", "swin", "mixed1", "mixed256", "int8out", "gather", "gatherl")


def measure_config(name: str, args, pk: dict, min_region_ms: float = 200.0, device_index: int = 0) -> dict:
    """One workload of another configuration, measured on the current device.

    The sequence of its problems runs back to back in one stream, captured as
    one CUDA graph of `reps` repetitions (no event inside: an event node between
    kernels serialises them), replayed inside the timed region while the clock
    sampler runs; reps is raised until the region lasts at least
    `min_region_ms`.  Per problem, our launch and the same-shape cuBLAS dense
    GEMM are timed by the same method (``_graph_us``)."""
    import structured_sparse_gemm_compress_b200 as nm

    if name == "single":
        ls, desc = inputs.single_layer(), "single ViT-B linear, INT8 2:4, T=197, 768->768, int32 out"
    elif name == "vitl":
        ls, desc = inputs.vit_l_fp16(), "ViT-L/16 linears, batch 32 (T=6304), FP16, N:M in {1:4,2:4,2:8}"
    elif name == "swin":
        ls, desc = inputs.swin_t_int8(), "Swin-T linears per stage, batch 128, INT8 + scale, N:M in {2:4,2:8}"
    elif name == "int8out":
        ls, desc = inputs.vit_b_int8(), ("ViT-B/16 INT8 linear set, batch 64 (T=12608), N:M in {1:4,2:4,2:8,4:8}, "
                                         "fused int8 output: per-channel scale + bias, GELU after fc1, requantised")
    elif name in ("mixed1", "mixed256"):
        T = 197 if name == "mixed1" else 50432
        ls, desc = inputs.vit_b_mixed(T), f"all 48 ViT-B linears at T={T}, per-layer N:M from {{dense,4:8,2:4,2:8,1:4}}"
    elif name == "gather":
        ls, desc = inputs.vit_b_int8(), ("ViT-B/16 INT8 linear set, batch 64 (T=12608), N:M in {1:4,2:4,2:8,4:8} with one "
                                         "pattern per 128-channel tile, activation feature-major, gather SpMM")
    elif name == "gatherl":
        ls, desc = inputs.vit_l_fp16(patterns=("1:4", "2:4", "2:8", "4:8")), (
            "ViT-L/16 linears, batch 32 (T=6304), FP16, N:M in {1:4,2:4,2:8,4:8} with one pattern per "
            "128-channel tile, activation feature-major, gather SpMM")
    else:
        raise SystemExit(f"unknown config {name}")
    if _ONLY:  # profiling one kernel shape of the config
        ls = [l for l in ls if f"{l.name}/{l.nm}" in _ONLY]
        if not ls:
            raise SystemExit(f"--only matched no problem of config {name}: {_ONLY}")
        desc = f"{desc}; only {','.join(_ONLY)}"
    stream = torch.cuda.current_stream()
    probs = []
    int8out = name == "int8out"
    gather = name in ("gather", "gatherl")
    for l in ls:
        W, X, sc = l.weight().cuda(), l.activation().cuda(), l.scale()
        sc = None if sc is None else sc.cuda()
        if gather:
            h = nm.nm_compress_tile(W, l.N, l.M)
            Xt = X.t().contiguous()
            Y = torch.empty((l.T, l.n_out), dtype=nm.out_dtype(h, sc is not None), device="cuda")
            call = (lambda st, h=h, Xt=Xt, Y=Y, sc=sc: nm.nm_spmm_gather(h, Xt, Y=Y, scale=sc, stream=st))
            probs.append((l, W, X, sc, h, Y, call))
            continue
        h = nm.nm_compress(W, l.N, l.M)
        if int8out:  # per-channel bias; GELU after fc1; one int8 step = 10 output units
            bias = inputs.normal_f32((l.n_out,), 5.0, l.seed + 3).cuda()
            act = "gelu" if l.name.endswith("fc1") else "none"
            Y = torch.empty((l.T, l.n_out), dtype=torch.int8, device="cuda")
            call = (lambda st, h=h, X=X, Y=Y, sc=sc, bias=bias, act=act:
                    nm.nm_spmm_ex(h, X, Y=Y, scale=sc, bias=bias, act=act, out="int8", out_scale=0.1, stream=st))
        else:
            Y = torch.empty((l.T, l.n_out), dtype=nm.out_dtype(h, sc is not None), device="cuda")
            call = (lambda st, h=h, X=X, Y=Y, sc=sc: nm.nm_spmm(h, X, Y=Y, scale=sc, stream=st))
        probs.append((l, W, X, sc, h, Y, call))
    torch.cuda.synchronize()

    def run_all(st):
        for p in probs:
            p[6](st)

    for _ in range(args.warmup):
        run_all(stream)
    torch.cuda.synchronize()

    def capture(n):
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
            for _ in range(n):
                run_all(cap)
        g.replay()
        torch.cuda.synchronize()
        return g

    # size the timed region: one replay of a single sequence gives the estimate
    g1 = capture(1)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g1.replay()
    b.record(stream)
    torch.cuda.synchronize()
    est_ms = max(a.elapsed_time(b), 1e-3)
    del g1
    reps = max(3, args.steps, int(min_region_ms / est_ms) + 1)
    chunk = min(reps, 200)  # graphs of at most 200 sequences, replayed back to back
    sizes = [chunk] * (reps // chunk) + ([reps % chunk] if reps % chunk else [])
    built = {n: capture(n) for n in sorted(set(sizes))}
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with NvmlSampler(device_index) as clk:
        torch.cuda.synchronize()
        clk.mark_start()
        a.record(stream)
        for n in sizes:
            built[n].replay()
        b.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    seq_ms = a.elapsed_time(b) / reps
    del built
    for h in (p[4] for p in probs):
        if nm.nm_device_status(h) != nm.NM_OK:
            raise RuntimeError(nm.nm_last_error())
    per = []
    for i, (l, W, X, sc, h, Y, call) in enumerate(probs):
        us = _graph_us(call, stream)
        rp = roofline_point(l, us, pk, 1 if int8out else None, int8out, gather)
        if not gather:
            plan = nm.nm_plan_query(h, l.T, scaled=sc is not None)
            rp["plan"] = {k: plan[k] for k in ("pair", "bn", "splits", "cluster", "grid")}
        if gather:  # the same weight with per-row patterns through nm_spmm (token-major X), same timing
            he = nm.nm_compress(W, l.N, l.M)
            Ye = torch.empty_like(Y)
            rp["per_row_patterns_us"] = round(_graph_us(lambda st: nm.nm_spmm(he, X, Y=Ye, scale=sc, stream=st),
                                                        stream), 2)
            he.destroy()
        # same-shape cuBLAS dense GEMM through torch, timed the same way (context)
        if l.dtype == inputs.INT8 and l.T > 16:
            Wt = W.t()
            fn = (lambda st, X=X, Wt=Wt: torch._int_mm(X, Wt))
        elif l.dtype != inputs.INT8:
            Wt = W.t()
            fn = (lambda st, X=X, Wt=Wt: torch.matmul(X, Wt))
        else:
            fn = None
        if fn is not None:
            cb = _graph_us(fn, stream)
            rp["cublas_dense_us"] = round(cb, 2)
            rp["vs_cublas"] = round(cb / us, 3)
        rp["problem"] = f"{l.name}/{l.nm}"
        rp["T,K,n_out"] = [l.T, l.K, l.n_out]
        per.append(rp)
    total_ops = sum(l.dense_ops() for l in ls)
    tot_roof = sum(p["roofline_us"] for p in per)
    line = {"config": {"workload": desc}, "metric": "dense-equivalent TOPS over the sequence", "unit": "TOPS",
            "value": total_ops / (seq_ms * 1e-3) / 1e12, "sequence_us": round(seq_ms * 1e3, 2),
            "useful_tops": sum(l.kept_ops() for l in ls) / (seq_ms * 1e-3) / 1e12,
            "sum_of_kernel_us": round(sum(p["us"] for p in per), 2),
            "per_problem_note": ("us: that launch alone, 20 back to back in a CUDA graph (median of 5 replays); "
                                 "cuBLAS timed the same way"),
            "roofline_us": round(tot_roof, 2), "roofline_frac": round(tot_roof / (seq_ms * 1e3), 3),
            "dtype": ls[0].dtype, "data": "synthetic", "launch": "CUDA graph of the sequence", "reps": reps,
            "clocks": clk.summary(), "per_problem": per}
    if any("cublas_dense_us" in p for p in per):
        line["cublas_dense_sum_us"] = round(sum(p.get("cublas_dense_us", 0.0) for p in per), 2)
    return line


def run_config(name: str, args) -> None:
    torch.cuda.set_device(0)
    pk = peaks()
    pk["int8_tops"] = measure_int8_peak(torch.device("cuda", 0))["int8_dense_tops"]
    line = measure_config(name, args, pk)
    line["int8_dense_peak_tops_measured"] = round(pk["int8_tops"], 1)
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU arm


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="nm", choices=["nm", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps eagerly")
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads' blocks in the default line")
    ap.add_argument("--config", default=None, choices=list(CONFIG_NAMES) + ["lut", "search", "cosearch"],
                    help="measure another workload (one JSON line) instead of the default ViT-B INT8 set")
    ap.add_argument("--only", action="append", default=[],
                    help="restrict to problems like vitb.fc1/2:4 (profiling a single kernel shape)")
    args = ap.parse_args()
    _ONLY.extend(args.only)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local_rank = rank_env()
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.config is not None:
        if rank == 0:
            {"lut": run_lut, "search": run_search, "cosearch": run_cosearch}.get(
                args.config, lambda a: run_config(args.config, a))(args)
        return

    import structured_sparse_gemm_compress_b200 as nm

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    def barrier():
        if dist is not None:
            dist.barrier()

    ls = layers()
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()

    # Host-side inputs (pinned) and device buffers.  Weights and activations are
    # shared by the four N:M variants of a layer; each problem has its own Y.
    host = {}
    for l in ls:
        if l.name not in host:
            host[l.name] = {"W": l.weight().pin_memory(), "X": l.activation().pin_memory(),
                            "s": l.scale().pin_memory()}
    devb = {n: {k: v.to(dev, non_blocking=True) for k, v in d.items()} for n, d in host.items()}
    handles, Ys = [], []
    for l in ls:
        handles.append(nm.nm_compress(devb[l.name]["W"], l.N, l.M))
        Ys.append(torch.empty((l.T, l.n_out), dtype=torch.float32, device=dev))
    torch.cuda.synchronize()

    pack_stream = torch.cuda.Stream()
    packed = [torch.cuda.Event() for _ in ls]  # re-pack of problem i done
    used = [torch.cuda.Event() for _ in ls]    # SpMM of problem i done (its packed image is free)

    def step(st=None, ps=None, first=True):
        """One pass over the 16 problems: per (layer, N:M) a re-pack of the weight
        on a second stream and the SpMM on the main stream.  The first step of a
        sequence re-packs after everything issued before it on the main stream
        (input copies, earlier work); a later step's re-pack of problem i waits
        only for the previous step's SpMM i, the one reader of that packed image.
        Each SpMM waits only for its own re-pack, so re-packs run under the
        SpMMs of other problems, across step boundaries too."""
        st = stream if st is None else st
        ps = pack_stream if ps is None else ps
        if first:
            ps.wait_stream(st)
        for i, l in enumerate(ls):
            if not first:
                ps.wait_event(used[i])
            nm.nm_recompress(handles[i], devb[l.name]["W"], stream=ps)
            packed[i].record(ps)
        for i, l in enumerate(ls):
            d = devb[l.name]
            st.wait_event(packed[i])
            nm.nm_spmm(handles[i], d["X"], Y=Ys[i], scale=d["s"], stream=st)
            used[i].record(st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for h in handles:
        if nm.nm_device_status(h) != nm.NM_OK:
            raise RuntimeError(nm.nm_last_error())

    # The K timed steps: CUDA graphs of up to 50 steps each (consecutive SpMMs
    # overlap launch and prologue through programmatic dependent launch),
    # replayed back to back so that exactly K steps run in the timed region,
    # after one untimed pass.  No event is recorded inside a graph: an event node
    # between two kernels serialises them and costs more than a short kernel.
    # --no-graph runs the steps eagerly.
    graphs, built = [], {}
    if not args.no_graph:
        chunk = min(args.steps, 50)
        sizes = [chunk] * (args.steps // chunk) + ([args.steps % chunk] if args.steps % chunk else [])
        for n in sorted(set(sizes)):
            g = torch.cuda.CUDAGraph()
            cap, cap_pack = torch.cuda.Stream(), torch.cuda.Stream()
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                for k in range(n):
                    step(st=cap, ps=cap_pack, first=k == 0)
            g.replay()  # upload + one untimed pass
            built[n] = g
        graphs = [built[n] for n in sizes]
        torch.cuda.synchronize()

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with NvmlSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        start.record(stream)
        if graphs:
            for g in graphs:
                g.replay()
                clk.poke()
        else:
            for k in range(args.steps):
                step(first=k == 0)
        stop.record(stream)
        clk.poke()
        torch.cuda.synchronize()
        clk.mark_end()
        barrier()
    ms_local = start.elapsed_time(stop)
    ms = max_over_ranks(ms_local, dist, dev)
    for h in handles:
        if nm.nm_device_status(h) != nm.NM_OK:
            raise RuntimeError(nm.nm_last_error())

    ops_step = sum(l.dense_ops() for l in ls)
    value = whole_job_tops(ops_step, args.steps, world, ms)
    useful = whole_job_tops(sum(l.kept_ops() for l in ls), args.steps, world, ms)

    # Roofline of the dominant kernel (the SpMM).  Its average launch duration is
    # the main stream's timed region (start/stop events on that stream) over the
    # 16*K SpMM launches it holds; the re-packs run on the side stream under
    # them.  That over-states the kernel's own duration (launch gaps, the first
    # re-pack of each step), so the fraction is a lower bound.
    spmm_bytes = sum(alg_bytes(l) for l in ls) * args.steps
    pk = peaks()
    achieved = spmm_bytes / (ms_local * 1e-3) / 1e9

    traffic = None
    tfile = os.path.join(ROOT, "profiles", "spmm_vitb_int8_traffic.json")
    if os.path.exists(tfile):
        tj = json.load(open(tfile))
        if tj.get("kernel_source_sha") == _kernel_sha():
            traffic = tj.get("bytes_per_launch")

    # Per-layer context (not the timed region), rank 0: every problem alone and
    # cuBLAS's dense int8 GEMM of the same shape (torch._int_mm, int32 out),
    # both timed by _graph_us (20 back-to-back launches in a CUDA graph, median
    # of 5 replays), plus the measured INT8 tensor peak.
    per_layer, cublas, pack_us, int8_peak = {}, {}, None, None
    if rank == 0:
        int8_peak = measure_int8_peak(dev)
        pk["int8_tops"] = int8_peak["int8_dense_tops"]
        for name in sorted({x.name for x in ls}):
            Xd, Wt = devb[name]["X"], devb[name]["W"].t()
            cublas[name] = _graph_us(lambda st, Xd=Xd, Wt=Wt: torch._int_mm(Xd, Wt), stream)
        for i, l in enumerate(ls):
            d = devb[l.name]
            us, p10, p90 = _graph_stats(
                lambda st, i=i, d=d: nm.nm_spmm(handles[i], d["X"], Y=Ys[i], scale=d["s"], stream=st), stream)
            rp = roofline_point(l, us, pk)
            rp["us_p10"], rp["us_p90"] = round(p10, 2), round(p90, 2)
            rp["hbm_frac"] = round(alg_bytes(l) / (us * 1e-6) / 1e9 / pk["hbm_gbs"], 3)
            rp["cublas_int8_dense_us"] = round(cublas[l.name], 2)
            rp["vs_cublas"] = round(cublas[l.name] / us, 3)
            plan = nm.nm_plan_query(handles[i], l.T, scaled=True)
            rp["plan"] = {k: plan[k] for k in ("pair", "bn", "splits", "cluster", "grid")}
            per_layer[f"{l.name}/{l.nm}"] = rp

        def all_packs(st):
            for i, l in enumerate(ls):
                nm.nm_recompress(handles[i], devb[l.name]["W"], stream=st)

        pack_us = _graph_us(all_packs, stream, reps=5)
        cublas = {k: {"us": round(v, 2), "dense_tops": round(
            next(x for x in ls if x.name == k).dense_ops() / v / 1e6, 1)} for k, v in cublas.items()}

    # End to end through the public API with host buffers: every step copies its
    # inputs (weights, activations, scales) from pinned host memory and reads
    # every output back.
    e2e = None
    if not args.no_e2e:
        yh = [torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True) for Y in Ys]
        h2d = sum(t.numel() * t.element_size() for d in host.values() for t in d.values())
        d2h = sum(y.numel() * y.element_size() for y in yh)
        e_steps = max(1, min(args.steps, 5))

        def e2e_step():
            for n, d in host.items():
                for key, t in d.items():
                    devb[n][key].copy_(t, non_blocking=True)
            step()
            for y, Y in zip(yh, Ys):
                y.copy_(Y, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(a.elapsed_time(b), dist, dev)
        e2e = {"value": whole_job_tops(ops_step, e_steps, world, ems), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        oracle.build()
        rows = args.cpu_rows or CPU_SAMPLE_ROWS
        secs, ops = cpu_oracle_run(ls, rows)
        cpu = {"value": ops / secs / 1e12, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
               "sample": f"first {rows} of 12608 tokens of each of the 16 (layer, N:M) problems "
                         f"(compress + decompress + triple-loop GEMM), {secs:.1f} s"}
        # the same oracle on one core, on an eighth of the sample
        all_threads = oracle.threads()
        oracle.set_threads(1)
        try:
            s1, o1 = cpu_oracle_run(ls, max(16, rows // 8))
        finally:
            oracle.set_threads(all_threads)
        cpu["one_core"] = {"value": o1 / s1 / 1e12, "unit": UNIT, "cores": 1,
                           "sample": f"first {max(16, rows // 8)} tokens of each problem, {s1:.1f} s"}

    del graphs, built
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    launches = 2 * len(ls) * args.steps  # one pack + one SpMM kernel per problem per step
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": WORKLOAD if not _ONLY else f"{WORKLOAD}; only {','.join(_ONLY)}",
                   "global_batch_tokens": 12608 * world, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2: each step streams ~1.7 GB",
                   "step": "per (layer, N:M): nm_recompress + nm_spmm",
                   "launch": "eager" if args.no_graph else "CUDA graphs of up to 50 steps replayed back to back"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                     "kernel": "nm_spmm kernels (streaming and CTA-pair variants): average launch = timed region / (16 K) launches on its stream", "peak_source": pk["source"]},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "useful_tops": useful,
        "spmm_launch_us_avg": 1e3 * ms_local / (args.steps * len(ls)),
        "pack_us_per_step": pack_us,
        "pack_overlapped": True,
        "int8_dense_peak_tops_measured": None if int8_peak is None else round(int8_peak["int8_dense_tops"], 1),
        "per_layer_note": ("each problem alone and cuBLAS's int8 GEMM of the same shape, both as 20 back-to-back "
                           "launches in a CUDA graph (ours: median and p10/p90 of 11 replays; cuBLAS: median of 5); "
                           "hbm_frac = algorithmic bytes / time / measured HBM; frac = roofline (max of HBM and "
                           "tensor time, INT8 peak measured) / time; useful_tops counts the kept weights only "
                           "((N/M) x dense-equivalent)"),
        "per_layer": per_layer,
        "cublas_int8_dense": cublas,
    }
    if not args.no_extras:
        # The other workloads, each with its own clock record (context for the
        # tensor-bound FP16 set, the small-token adaptive split-K and the
        # Swin stages): the sequence timed as one graph, per problem ours and
        # cuBLAS's timed the same way.
        import types
        eargs = types.SimpleNamespace(steps=3, warmup=3)
        extras = {}
        for cname in ("vitl", "mixed1", "single", "swin", "mixed256"):
            r = measure_config(cname, eargs, pk, min_region_ms=200.0, device_index=local_rank)
            for p in r["per_problem"]:
                p.pop("T,K,n_out", None)
            extras[cname] = r
        line["configs"] = extras
    print(json.dumps(line), flush=True)


def _kernel_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("nm_spmm.cu", "nm_device.cuh", "nm_api.cu"):  # the kernels and the planner that picks them
        h.update(open(os.path.join(ROOT, "structured_sparse_gemm_compress_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
