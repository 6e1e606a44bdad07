"""Latency-constrained layer-wise N:M search.

"Realizable N:M Sparse Transformer Inference via Search-Kernel Co-Design"
(arXiv 2607.12505), sections 1 and 3: given a model and an end-to-end latency
budget, choose one N:M pattern per linear layer; a calibrated LUT latency
predictor enforces feasibility and a feasible-region-aware evolutionary solver
explores the (fragmented) feasible region.  The pages give no more detail and
the accuracy objective needs trained weights and ImageNet-1K, which are not
available here, so this module takes the plainest reading with a proxy:

* quality of a configuration = the fraction of the model's total weight
  magnitude (sum of |w|) that the chosen patterns keep;
* latency = the calibrated LUT prediction (``lut.LatencyLUT.predict``);
* solver = a genetic algorithm whose infeasible offspring are repaired onto
  the feasible region: while over budget, apply the single-layer move to a
  faster pattern with the best latency saved per quality lost;
* ``solve_exact`` solves the same separable problem (a multiple-choice
  knapsack) by dynamic programming over discretised latency, so the
  evolutionary result can be checked against the optimum.
"""
from __future__ import annotations

import random
from dataclasses import dataclass

import numpy as np

from .lut import TILE_PATTERNS


@dataclass
class Problem:
    """lat[l][p] (us, calibrated per-layer latency), keep[l][p] (kept |w| mass),
    total mass, and the budget on the calibrated sequence latency."""
    patterns: list[str]
    lat: np.ndarray      # [L, P]
    keep: np.ndarray     # [L, P]
    total_mass: float
    offset: float        # calibrated constant (b * layers)
    budget: float

    def latency(self, a: np.ndarray) -> float:
        return float(self.lat[np.arange(len(a)), a].sum() + self.offset)

    def quality(self, a: np.ndarray) -> float:
        return float(self.keep[np.arange(len(a)), a].sum() / self.total_mass)

    def feasible(self, a: np.ndarray) -> bool:
        return self.latency(a) <= self.budget + 1e-9


def make_problem(layers, lut_, T: int, keep_mass: dict, total_mass: dict, budget_us: float,
                 patterns=None) -> Problem:
    """Per-layer latency from the calibrated LUT (a * table entry, plus c for a
    tile-shared pattern) and the constant b * layers; keep_mass[(layer name,
    pattern)] kept |w| mass."""
    patterns = list(patterns) if patterns else sorted({k[2] for k in lut_.table})
    L, P = len(layers), len(patterns)
    c = getattr(lut_, "c", 0.0)
    lat = np.array([[lut_.a * lut_.lookup(l.K, l.n_out, p, T) + (c if p in TILE_PATTERNS else 0.0)
                     for p in patterns] for l in layers])
    keep = np.array([[keep_mass[(l.name, p)] for p in patterns] for l in layers], dtype=np.float64)
    tot = float(sum(total_mass[l.name] for l in layers))
    return Problem(patterns, lat, keep, tot, lut_.b * L, float(budget_us))


def repair(prob: Problem, a: np.ndarray) -> np.ndarray | None:
    """Move layers to faster patterns, best latency-saved per quality-lost
    first, until the configuration meets the budget; None if it cannot."""
    a = a.copy()
    L = len(a)
    while not prob.feasible(a):
        cur_lat = prob.lat[np.arange(L), a]
        cur_keep = prob.keep[np.arange(L), a]
        saved = cur_lat[:, None] - prob.lat          # [L, P] latency saved by switching
        lost = cur_keep[:, None] - prob.keep         # [L, P] quality lost
        ok = saved > 1e-12
        if not ok.any():
            return None
        ratio = np.where(ok, saved / np.maximum(lost, 1e-12), -np.inf)
        l, p = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        a[l] = p
    return a


def solve_greedy(prob: Problem) -> np.ndarray | None:
    """Start from the best-quality pattern of every layer and repair."""
    return repair(prob, np.argmax(prob.keep, axis=1))


def solve_evolutionary(prob: Problem, pop: int = 64, generations: int = 150, seed: int = 0,
                       elite: int = 4, tournament: int = 3) -> np.ndarray | None:
    """Genetic search with tournament selection, uniform crossover, per-gene
    mutation and repair onto the feasible region; returns the best feasible
    configuration found (at least as good as the greedy one it is seeded with)."""
    rng = random.Random(seed)
    L, P = prob.lat.shape
    fitness = lambda a: prob.quality(a)   # every member is feasible after repair
    members = []
    g = solve_greedy(prob)
    if g is not None:
        members.append(g)
    tries = 0
    while len(members) < pop and tries < 20 * pop:
        tries += 1
        r = repair(prob, np.array([rng.randrange(P) for _ in range(L)]))
        if r is not None:
            members.append(r)
    if not members:
        return None
    for _ in range(generations):
        members.sort(key=fitness, reverse=True)
        nxt = [m.copy() for m in members[:elite]]

        def pick():
            c = [members[rng.randrange(len(members))] for _ in range(tournament)]
            return max(c, key=fitness)

        while len(nxt) < pop:
            pa, pb = pick(), pick()
            child = np.where(np.array([rng.random() < 0.5 for _ in range(L)]), pa, pb)
            for i in range(L):
                if rng.random() < 1.0 / L:
                    child[i] = rng.randrange(P)
            child = repair(prob, child)
            if child is not None:
                nxt.append(child)
        members = nxt
    return max(members, key=fitness)


def polish(prob: Problem, a: np.ndarray) -> np.ndarray:
    """Single-layer moves into the unrounded slack: while some one-layer change
    raises the quality and keeps the exact latency within the budget, apply the
    one that raises it most."""
    a = a.copy()
    L = len(a)
    while True:
        lat = prob.latency(a)
        cur_keep = prob.keep[np.arange(L), a]
        cur_lat = prob.lat[np.arange(L), a]
        gain = prob.keep - cur_keep[:, None]                      # [L, P]
        fits = lat - cur_lat[:, None] + prob.lat <= prob.budget + 1e-9
        gain = np.where(fits & (gain > 1e-12), gain, -np.inf)
        l, p = np.unravel_index(int(np.argmax(gain)), gain.shape)
        if not np.isfinite(gain[l, p]):
            return a
        a[l] = p


def solve_exact(prob: Problem, resolution_us: float = 0.05) -> np.ndarray | None:
    """Optimum of the multiple-choice knapsack by dynamic programming over
    latency in steps of ``resolution_us`` (latencies rounded up, so the result
    is feasible; it is optimal up to that rounding), then ``polish`` into the
    slack the rounding left."""
    L, P = prob.lat.shape
    cap = int(np.floor((prob.budget - prob.offset) / resolution_us + 1e-9))
    if cap < 0:
        return None
    w = np.ceil(prob.lat / resolution_us - 1e-9).astype(np.int64)
    cap = min(cap, int(w.max(axis=1).sum()))  # no configuration is slower than this
    NEG = -np.inf
    best = np.full(cap + 1, NEG)
    best[0] = 0.0
    choice = np.zeros((L, cap + 1), dtype=np.int16)
    for l in range(L):
        nb = np.full(cap + 1, NEG)
        for p in range(P):
            wl = w[l, p]
            if wl > cap:
                continue
            cand = np.full(cap + 1, NEG)
            cand[wl:] = best[:cap + 1 - wl] + prob.keep[l, p]
            upd = cand > nb
            nb[upd] = cand[upd]
            choice[l, upd] = p
        best = nb
    if not np.isfinite(best).any():
        return None
    c = int(np.argmax(best))
    a = np.zeros(L, dtype=np.int64)
    for l in range(L - 1, -1, -1):
        a[l] = choice[l, c]
        c -= w[l, a[l]]
    return polish(prob, a)


def kept_mass(W, N: int, M: int, tile: bool = False) -> float:
    """Sum of |w| over the weights the library's compressor keeps (GPU): the
    values exported from an ``nm_compress`` handle (``nm_compress_tile`` when
    ``tile``: one pattern per 128 output channels)."""
    import torch

    import structured_sparse_gemm_compress_b200 as nm
    h = nm.nm_compress_tile(W, N, M) if tile else nm.nm_compress(W, N, M)
    values, _ = nm.nm_export(h)
    h.destroy()
    return float(values.to(torch.float64).abs().sum())
