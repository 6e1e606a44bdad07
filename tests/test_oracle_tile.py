"""Pins for the oracle's tile-shared (vector-wise) compress.

The rule: rows in tiles of V consecutive rows share one pattern; in every group
of M positions a tile keeps the N positions of largest column mass (sum of |w|
over the tile's rows), ties to the lower position.  Pinned by hand-worked
examples (tests/golden/tile_hand.json), brute-force enumeration of the subsets
of largest mass, the V = 1 reduction to the per-row rule (itself pinned in
test_oracle.py), invariants, and an fp16 case that single-precision sums would
decide the other way.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tile_hand.json")
PATTERNS = [(1, 4), (2, 4), (2, 8), (4, 8)]


def _positions(idx, n_groups, N, M):
    """Global k positions per row decoded from the canonical 4-bit stream."""
    out = []
    for r in range(idx.shape[0]):
        row = []
        for e in range(n_groups * N):
            b = int(idx[r, e // 2])
            p = (b >> 4) if (e & 1) else (b & 0xF)
            row.append((e // N) * M + p)
        out.append(row)
    return out


def _best_subset(scores, N):
    """N-subset of largest total score, then lexicographically smallest."""
    best = None
    for sub in itertools.combinations(range(len(scores)), N):
        key = (-sum(scores[p] for p in sub), sub)
        if best is None or key < best:
            best = key
    return list(best[1])


def _brute_force_tile_positions(mag, V, N, M):
    """Per row: the positions its tile keeps, by enumeration over subsets."""
    n, k = mag.shape
    out = []
    for r in range(n):
        t0 = (r // V) * V
        rows = mag[t0:min(t0 + V, n)]
        pos = []
        for g in range(k // M):
            scores = [sum(rows[:, g * M + p]) for p in range(M)]
            pos += [g * M + p for p in _best_subset(scores, N)]
        out.append(pos)
    return out


# --------------------------------------------------------------------------- golden


def _case_params(name):
    v, nm = name.split()
    return int(v[2:]), *map(int, nm.split(":"))


@pytest.mark.parametrize("name", sorted(json.load(open(GOLDEN))["cases"]))
def test_tile_hand_examples(name):
    g = json.load(open(GOLDEN))
    case = g["cases"][name]
    V, N, M = _case_params(name)
    W = np.array(g["W"], dtype=np.int8)
    values, idx = oracle.compress_tile(W, N, M, tile=V)
    assert values.reshape(W.shape[0], -1).tolist() == case["values"]
    pos = _positions(idx, W.shape[1] // M, N, M)
    for r in range(W.shape[0]):
        assert pos[r] == case["tile_positions"][r // V]
    if "Y" in case:
        X = np.array(g["X"], dtype=np.int8)
        Wm = oracle.decompress(values, idx, W.shape[0], W.shape[1], N, M)
        assert oracle.gemm(X, Wm).tolist() == case["Y"]


def test_tile_hand_fixture_is_consistent():
    """The fixture's scores are the column sums of |W|, and its kept sets are
    the best subsets of those scores (checks the hand work itself)."""
    g = json.load(open(GOLDEN))
    W = np.abs(np.array(g["W"], dtype=np.int64))
    assert g["scores"]["V=2"]["rows 0-1"] == W[0:2].sum(0).tolist()
    assert g["scores"]["V=2"]["rows 2-3"] == W[2:4].sum(0).tolist()
    assert g["scores"]["V=4"]["rows 0-3"] == W.sum(0).tolist()
    for name, case in g["cases"].items():
        V, N, M = _case_params(name)
        want = _brute_force_tile_positions(W, V, N, M)
        for r in range(W.shape[0]):
            assert case["tile_positions"][r // V] == want[r]


# --------------------------------------------------------------------------- rule


@pytest.mark.parametrize("V", [1, 2, 3, 5])
@pytest.mark.parametrize("N,M", PATTERNS)
def test_tile_brute_force_int8(N, M, V):
    rng = np.random.default_rng(31 + V)
    W = rng.integers(-3, 4, size=(11, 4 * M), dtype=np.int8)  # ties everywhere; ragged last tile
    values, idx = oracle.compress_tile(W, N, M, tile=V)
    pos = _positions(idx, W.shape[1] // M, N, M)
    want = _brute_force_tile_positions(np.abs(W.astype(np.int64)), V, N, M)
    assert pos == want
    for r in range(W.shape[0]):
        assert values[r].reshape(-1).tolist() == [int(W[r, c]) for c in want[r]]


@pytest.mark.parametrize("N,M", PATTERNS)
def test_tile_brute_force_fp16(N, M):
    rng = np.random.default_rng(41)
    base = rng.choice([0.0, -0.0, 0.5, -0.5, 1.0, -1.5, 2.0, 3.0e-5, -6.0e-8], size=(9, 3 * M))
    W = torch.tensor(base, dtype=torch.float32).to(torch.float16).numpy()
    values, idx = oracle.compress_tile(W, N, M, tile=4)
    pos = _positions(idx, W.shape[1] // M, N, M)
    mag = [[abs(float(x)) for x in row] for row in W.astype(np.float64)]
    want = _brute_force_tile_positions(np.array(mag, dtype=object), 4, N, M)
    assert pos == want
    for r in range(W.shape[0]):
        assert values[r].reshape(-1).view(np.uint16).tolist() == [W[r, c].view(np.uint16).item() for c in want[r]]


@pytest.mark.parametrize("dtype", [np.int8, np.float16])
@pytest.mark.parametrize("N,M", PATTERNS + [(4, 4)])
def test_tile_of_one_row_is_the_row_rule(N, M, dtype):
    rng = np.random.default_rng(51)
    if dtype == np.int8:
        W = rng.integers(-5, 6, size=(20, 8 * M), dtype=np.int8)
    else:
        W = (rng.standard_normal((20, 8 * M)) * 0.02).astype(np.float16)
    vt, it = oracle.compress_tile(W, N, M, tile=1)
    vr, ir = oracle.compress(W, N, M)
    assert np.array_equal(vt.view(np.uint8), vr.view(np.uint8)) and np.array_equal(it, ir)


def test_tile_fp16_scores_are_exact():
    """2048 + 2^-24 beats 2048: a single-precision running sum rounds the small
    term away and would keep the lower position instead."""
    tiny = np.float16(2.0 ** -24)
    assert float(tiny) == 2.0 ** -24
    W = np.zeros((3, 4), dtype=np.float16)
    W[:, 0] = [1024, 1024, 0]          # mass 2048
    W[:, 1] = [2048, tiny, tiny]       # mass 2048 + 2^-23
    W[:, 2] = [-1024, -1023.5, 0]      # mass 2047.5
    f32 = np.float32(0)
    for x in W[:, 1]:
        f32 = np.float32(f32 + np.float32(x))
    assert f32 == np.float32(2048)     # the rounding the exact rule must avoid
    _, idx = oracle.compress_tile(W, 1, 4, tile=3)
    assert _positions(idx, 1, 1, 4) == [[1], [1], [1]]
    _, idx2 = oracle.compress_tile(W, 2, 4, tile=3)
    assert _positions(idx2, 1, 2, 4) == [[0, 1]] * 3


@pytest.mark.parametrize("N,M", PATTERNS + [(8, 8)])
def test_tile_invariants(N, M):
    rng = np.random.default_rng(61)
    n_out, k, V = 300, 24 * M, 128
    W = rng.integers(-127, 128, size=(n_out, k), dtype=np.int8)
    values, idx = oracle.compress_tile(W, N, M, tile=V)
    pos = _positions(idx, k // M, N, M)
    for t0 in range(0, n_out, V):
        rows = pos[t0:min(t0 + V, n_out)]
        assert all(p == rows[0] for p in rows)             # one pattern per tile
    for r in range(n_out):
        assert all(b > a for a, b in zip(pos[r], pos[r][1:]))  # ascending, distinct
        assert values[r].reshape(-1).tolist() == [int(W[r, c]) for c in pos[r]]
    if N == M:
        assert pos[0] == list(range(k))
    # the decompressed weight has at most N non-zeros in every group
    Wm = oracle.decompress(values, idx, n_out, k, N, M)
    assert np.count_nonzero(Wm.reshape(n_out, k // M, M), axis=2).max() <= N


def test_tile_rejects_bf16_and_bad_arguments():
    W16 = np.zeros((4, 8), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.compress_tile(W16, 2, 4, tile=2, dtype="bf16")
    W = np.zeros((4, 8), dtype=np.int8)
    for bad in (0, -1, 4097):
        with pytest.raises(ValueError):
            oracle.compress_tile(W, 2, 4, tile=bad)
    with pytest.raises(ValueError):
        oracle.compress_tile(np.zeros((4, 6), dtype=np.int8), 2, 4, tile=2)
