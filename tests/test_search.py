"""Latency-constrained layer-wise N:M search (host logic, no GPU): the exact
solver against brute force, the evolutionary solver against the exact one."""
import itertools

import numpy as np
import pytest

from structured_sparse_gemm_compress_b200 import search


def _problem(L, P, seed, budget_frac, integer=False):
    rng = np.random.default_rng(seed)
    base = rng.uniform(5, 50, size=(L, 1))
    speed = np.sort(rng.uniform(0.4, 1.0, size=(L, P)), axis=1)[:, ::-1]   # pattern 0 slowest
    lat = base * speed
    if integer:
        lat = np.round(lat * 20) / 20  # multiples of the DP resolution
    keep = base * np.sort(rng.uniform(0.3, 1.0, size=(L, P)), axis=1)[:, ::-1]  # slower keeps more
    total = float(base.sum() * 1.0)
    lo, hi = lat.min(axis=1).sum(), lat.max(axis=1).sum()
    return search.Problem([f"p{i}" for i in range(P)], lat, keep, total, 2.0, lo + 2.0 + budget_frac * (hi - lo))


@pytest.mark.parametrize("seed", range(6))
def test_exact_solver_matches_brute_force(seed):
    prob = _problem(4, 5, seed, 0.4, integer=True)
    best, arg = -1.0, None
    for a in itertools.product(range(5), repeat=4):
        a = np.array(a)
        if prob.feasible(a) and prob.quality(a) > best:
            best, arg = prob.quality(a), a
    got = search.solve_exact(prob)
    assert prob.feasible(got)
    assert prob.quality(got) == pytest.approx(best, rel=1e-12)


@pytest.mark.parametrize("seed", range(3))
def test_evolutionary_reaches_the_optimum_region(seed):
    prob = _problem(48, 5, 100 + seed, 0.35)
    ex = search.solve_exact(prob, resolution_us=0.01)
    ga = search.solve_evolutionary(prob, pop=48, generations=120, seed=seed)
    gr = search.solve_greedy(prob)
    for a in (ex, ga, gr):
        assert a is not None and prob.feasible(a)
    assert prob.quality(ga) >= prob.quality(gr) - 1e-12          # seeded with the greedy solution
    assert prob.quality(ga) >= 0.998 * prob.quality(ex)
    assert prob.quality(ex) >= prob.quality(ga) - 1e-6           # the exact solver is an upper bound
    # (up to its latency rounding, which only makes it more conservative)


def test_repair_and_infeasible_budgets():
    prob = _problem(8, 5, 7, 0.0)
    fastest = np.argmin(prob.lat, axis=1)
    assert prob.feasible(fastest)
    prob.budget = prob.latency(fastest) - 1.0
    assert search.repair(prob, np.zeros(8, dtype=np.int64)) is None
    assert search.solve_exact(prob) is None
    assert search.solve_evolutionary(prob, pop=8, generations=2) is None


def test_unconstrained_budget_keeps_best_quality():
    prob = _problem(10, 5, 9, 1.0)
    prob.budget = 1e9
    for a in (search.solve_greedy(prob), search.solve_exact(prob), search.solve_evolutionary(prob, pop=16, generations=10)):
        assert prob.quality(a) == pytest.approx(prob.keep.max(axis=1).sum() / prob.total_mass)


def test_exact_solver_recovers_what_rounding_hides():
    """Two layers whose exact latencies fill the budget exactly: rounding every
    latency up would make the best pair look infeasible; the polish restores it."""
    prob = search.Problem(["fast", "good"], np.array([[1.0, 1.02], [1.0, 1.03]]),
                          np.array([[1.0, 2.0], [1.0, 2.0]]), total_mass=4.0, offset=0.0, budget=2.03)
    a = search.solve_exact(prob, resolution_us=0.05)
    assert prob.feasible(a)
    assert prob.quality(a) == pytest.approx(3.0 / 4.0)      # one layer upgraded within 2.03
    unpolished_best = max(prob.quality(np.array(x)) for x in ([0, 0], [1, 0], [0, 1], [1, 1])
                          if prob.latency(np.array(x)) <= 2.03 + 1e-9)
    assert prob.quality(a) == pytest.approx(unpolished_best)


def test_polish_never_breaks_the_budget():
    rng = np.random.default_rng(3)
    for _ in range(50):
        L, P = 6, 4
        lat = rng.uniform(1.0, 3.0, (L, P))
        keep = rng.uniform(0.0, 1.0, (L, P))
        budget = float(lat.min(axis=1).sum() + rng.uniform(0.0, 3.0))
        prob = search.Problem([str(i) for i in range(P)], lat, keep, 10.0, 0.0, budget)
        a = search.polish(prob, np.argmin(lat, axis=1))
        assert prob.feasible(a)
        assert prob.quality(a) >= prob.quality(np.argmin(lat, axis=1)) - 1e-12
