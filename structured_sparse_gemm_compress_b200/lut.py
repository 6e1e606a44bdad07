"""Calibrated lookup-table (LUT) latency predictor for layer-wise N:M sequences.

"Realizable N:M Sparse Transformer Inference via Search-Kernel Co-Design"
(arXiv 2607.12505), sections 1 and 3: the layer-wise N:M search relies on a
calibrated, profiling-based LUT latency predictor that keeps candidate
configurations inside the deployment latency budget.  The pages give no more
detail, so this module takes the plainest reading:

* the table holds the measured latency of one ``nm_spmm`` launch for every
  (K, n_out, pattern, T) profiled on the target GPU; between profiled token
  counts the latency is interpolated linearly in T (extrapolated from the two
  nearest points outside the profiled range);
* a configuration (one pattern per linear layer) is predicted by summing its
  layers' table entries, then calibrated against measured end-to-end sequence
  latencies with a least-squares fit
      measured ~ a * sum + b * layers + c * tile-shared layers
  (a absorbs overlap and cache effects between back-to-back launches, b a
  fixed cost per launch, c what a tile-shared gather launch costs in a
  sequence beyond its isolated table entry; c is fitted only when the samples
  contain such layers, else 0).

Profiling and sequence timing run the product kernels through the package's
binding; the table logic itself is plain host code.
"""
from __future__ import annotations

import json
import random
from dataclasses import dataclass

import numpy as np

PATTERNS = {"dense": (4, 4), "4:8": (4, 8), "2:4": (2, 4), "2:8": (2, 8), "1:4": (1, 4)}
# One pattern per 128 output channels (nm_compress_tile), run through the
# activation gather (nm_spmm_gather, activation given feature-major): the
# kernel side of the search-kernel co-design offers these as further choices.
TILE_PATTERNS = {"t4:8": (4, 8), "t2:8": (2, 8), "t1:4": (1, 4)}


def n_tile_layers(assignment: list[str]) -> int:
    """How many layers of an assignment use a tile-shared pattern."""
    return sum(1 for p in assignment if p in TILE_PATTERNS)


def pattern_nm(pattern: str) -> tuple[int, int, bool]:
    """(N, M, tile-shared) of a pattern name from PATTERNS or TILE_PATTERNS."""
    if pattern in PATTERNS:
        return (*PATTERNS[pattern], False)
    if pattern in TILE_PATTERNS:
        return (*TILE_PATTERNS[pattern], True)
    raise KeyError(f"unknown pattern {pattern!r}")


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer: Y[T, n_out] = X[T, K] . W[n_out, K]^T."""
    name: str
    K: int
    n_out: int


def vit_b_layers(blocks: int = 12) -> list[LayerSpec]:
    """The 4 linears of each ViT-B/16 block (qkv, proj, fc1, fc2)."""
    out = []
    for b in range(blocks):
        out += [LayerSpec(f"b{b}.qkv", 768, 2304), LayerSpec(f"b{b}.proj", 768, 768),
                LayerSpec(f"b{b}.fc1", 768, 3072), LayerSpec(f"b{b}.fc2", 3072, 768)]
    return out


def random_assignment(n_layers: int, seed: int, patterns=tuple(PATTERNS)) -> list[str]:
    rng = random.Random(seed)
    return [rng.choice(patterns) for _ in range(n_layers)]


def stratified_assignments(n_layers: int, seed: int, per_row=tuple(PATTERNS),
                           tile=tuple(TILE_PATTERNS), fractions=(0.0, 0.25, 0.5, 0.75, 1.0)) -> list[list[str]]:
    """Calibration assignments whose share of tile-shared layers is set on
    purpose (one assignment per fraction, layers and patterns drawn at random),
    so that a per-family term of the calibration is identifiable."""
    rng = random.Random(seed)
    out = []
    for f in fractions:
        k = round(f * n_layers)
        tiled = set(rng.sample(range(n_layers), k))
        out.append([rng.choice(tile) if i in tiled else rng.choice(per_row) for i in range(n_layers)])
    return out


class LatencyLUT:
    """Measured per-launch latency table plus the sequence calibration."""

    def __init__(self, table: dict[tuple[int, int, str, int], float], meta: dict | None = None,
                 a: float = 1.0, b: float = 0.0, c: float = 0.0):
        self.table = dict(table)
        self.meta = dict(meta or {})
        self.a, self.b, self.c = float(a), float(b), float(c)

    # ---------------------------------------------------------------- lookup
    def lookup(self, K: int, n_out: int, pattern: str, T: int) -> float:
        """Latency (us) of one launch; linear in T between profiled token counts."""
        pts = sorted((t, us) for (k, n, p, t), us in self.table.items() if (k, n, p) == (K, n_out, pattern))
        if not pts:
            raise KeyError(f"no entry for K={K} n_out={n_out} pattern={pattern}")
        ts = [t for t, _ in pts]
        if T in ts:
            return pts[ts.index(T)][1]
        if len(pts) == 1:
            raise KeyError(f"only T={ts[0]} profiled for K={K} n_out={n_out} pattern={pattern}")
        i = int(np.searchsorted(ts, T))
        i = min(max(i, 1), len(pts) - 1)   # bracketing pair, or the two nearest at an end
        (t0, u0), (t1, u1) = pts[i - 1], pts[i]
        return u0 + (u1 - u0) * (T - t0) / (t1 - t0)

    def raw_sum(self, layers: list[LayerSpec], assignment: list[str], T: int) -> float:
        if len(layers) != len(assignment):
            raise ValueError("one pattern per layer")
        return sum(self.lookup(l.K, l.n_out, p, T) for l, p in zip(layers, assignment))

    def predict(self, layers: list[LayerSpec], assignment: list[str], T: int) -> float:
        """Calibrated end-to-end latency (us) of the layer sequence."""
        return (self.a * self.raw_sum(layers, assignment, T) + self.b * len(layers)
                + self.c * n_tile_layers(assignment))

    # ---------------------------------------------------------------- calibration
    def calibrate(self, samples: list[tuple[list[LayerSpec], list[str], int, float]]) -> tuple[float, float]:
        """Least-squares fit of measured ~ a * raw_sum + b * n_layers
        (+ c * n_tile_layers when any sample has tile-shared layers) over
        (layers, assignment, T, measured_us) samples; sets a, b, c and returns (a, b)."""
        A = np.array([[self.raw_sum(ls, asg, T), float(len(ls)), float(n_tile_layers(asg))]
                      for ls, asg, T, _ in samples])
        y = np.array([m for *_, m in samples])
        self.c = 0.0
        if A[:, 2].any() and len(samples) >= 3 and np.linalg.matrix_rank(A) == 3:
            sol, *_ = np.linalg.lstsq(A, y, rcond=None)
            self.a, self.b, self.c = float(sol[0]), float(sol[1]), float(sol[2])
        elif len(samples) >= 2 and np.linalg.matrix_rank(A[:, :2]) == 2:
            sol, *_ = np.linalg.lstsq(A[:, :2], y, rcond=None)
            self.a, self.b = float(sol[0]), float(sol[1])
        else:  # one sample (or all with the same layer count and sum): scale only
            self.a, self.b = float(y.sum() / A[:, 0].sum()), 0.0
        return self.a, self.b

    # ---------------------------------------------------------------- persistence
    def to_json(self) -> str:
        rows = [{"K": k, "n_out": n, "pattern": p, "T": t, "us": us} for (k, n, p, t), us in sorted(self.table.items())]
        return json.dumps({"meta": self.meta, "calibration": {"a": self.a, "b": self.b, "c": self.c},
                           "entries": rows}, indent=1)

    @staticmethod
    def from_json(text: str) -> "LatencyLUT":
        d = json.loads(text)
        table = {(r["K"], r["n_out"], r["pattern"], r["T"]): float(r["us"]) for r in d["entries"]}
        cal = d.get("calibration", {})
        return LatencyLUT(table, d.get("meta"), cal.get("a", 1.0), cal.get("b", 0.0), cal.get("c", 0.0))


# -------------------------------------------------------------------- GPU side

def _graph_time_us(launch, reps: int) -> float:
    """Average time (us) of one call of ``launch(stream)`` over ``reps`` calls
    captured back to back in one CUDA graph, after warm-up; events only around
    the whole replay."""
    import torch

    for _ in range(3):
        launch(None)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
        for _ in range(reps):
            launch(cap)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / reps
    del g
    return us


class _Workspace:
    """Seeded device operands per (K, n_out) and per T, reused across patterns."""

    def __init__(self, seed: int = 11):
        self.seed = seed
        self.W, self.X, self.s = {}, {}, {}

    def weight(self, K, n_out):
        import torch

        from . import inputs
        if (K, n_out) not in self.W:
            self.W[(K, n_out)] = inputs.int8_uniform((n_out, K), -127, 127, self.seed + K + n_out).cuda()
            self.s[(K, n_out)] = inputs.scale_uniform(n_out, 0.001, 0.01, self.seed + 2 * K + n_out).cuda()
        return self.W[(K, n_out)], self.s[(K, n_out)]

    def act(self, T, K):
        from . import inputs
        if (T, K) not in self.X:
            self.X[(T, K)] = inputs.int8_uniform((T, K), -128, 127, self.seed + T + K).cuda()
        return self.X[(T, K)]

    def act_t(self, T, K):
        """The same activation, feature-major [K, T] (the gather's layout)."""
        if ("t", T, K) not in self.X:
            self.X[("t", T, K)] = self.act(T, K).t().contiguous()
        return self.X[("t", T, K)]


def _handle_and_call(W, s, ws: "_Workspace", pattern: str, T: int, K: int, Y):
    """Compress W for `pattern` and return (handle, launch(stream)) of one SpMM."""
    import structured_sparse_gemm_compress_b200 as nm
    N, M, tile = pattern_nm(pattern)
    if tile:
        h = nm.nm_compress_tile(W, N, M)
        Xt = ws.act_t(T, K)
        return h, (lambda st: nm.nm_spmm_gather(h, Xt, Y=Y, scale=s, stream=st))
    h = nm.nm_compress(W, N, M)
    X = ws.act(T, K)
    return h, (lambda st: nm.nm_spmm(h, X, Y=Y, scale=s, stream=st))


def profile(shapes: list[tuple[int, int]], patterns: list[str], Ts: list[int], reps: int = 20,
            ws: _Workspace | None = None) -> LatencyLUT:
    """Profile one SpMM launch (INT8, per-channel scale, fp32 output) for every
    (K, n_out) in ``shapes``, pattern and token count on the current GPU:
    ``nm_spmm`` for PATTERNS, ``nm_spmm_gather`` for TILE_PATTERNS."""
    import torch

    ws = ws or _Workspace()
    table = {}
    for K, n_out in shapes:
        W, s = ws.weight(K, n_out)
        for p in patterns:
            for T in Ts:
                Y = torch.empty((T, n_out), dtype=torch.float32, device="cuda")
                h, call = _handle_and_call(W, s, ws, p, T, K, Y)
                table[(K, n_out, p, T)] = _graph_time_us(call, reps)
                h.destroy()
    meta = {"device": torch.cuda.get_device_name(), "reps": reps, "dtype": "int8", "output": "fp32 scaled"}
    return LatencyLUT(table, meta)


def measure_sequence(layers: list[LayerSpec], assignment: list[str], T: int, reps: int = 5,
                     ws: _Workspace | None = None) -> float:
    """Measured latency (us) of the whole layer sequence, launched back to back
    in one stream (one CUDA graph of ``reps`` passes, events around it)."""
    import torch

    ws = ws or _Workspace()
    handles, calls = [], []
    for l, p in zip(layers, assignment):
        W, s = ws.weight(l.K, l.n_out)
        Y = torch.empty((T, l.n_out), dtype=torch.float32, device="cuda")
        h, call = _handle_and_call(W, s, ws, p, T, l.K, Y)
        handles.append((h, Y))
        calls.append(call)

    def one_pass(st):
        for call in calls:
            call(st)

    us = _graph_time_us(one_pass, reps)
    for h, _ in handles:
        h.destroy()
    return us
