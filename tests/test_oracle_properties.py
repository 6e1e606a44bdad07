"""Property-based pins of the oracle (hypothesis): for random small int8
weights with many ties, the per-row and tile-shared compressors agree with
brute-force enumeration of the best subsets, the decompressed weight keeps
exactly the chosen entries, and the GEMM over it equals numpy's int64 product."""
import itertools

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

PATTERNS = [(1, 4), (2, 4), (2, 8), (4, 8), (4, 4)]


def _best(scores, N):
    return min(itertools.combinations(range(len(scores)), N), key=lambda sub: (-sum(scores[p] for p in sub), sub))


def _positions(idx, groups, N, M):
    out = []
    for r in range(idx.shape[0]):
        row = []
        for e in range(groups * N):
            b = int(idx[r, e // 2])
            row.append((e // N) * M + ((b >> 4) if e & 1 else (b & 0xF)))
        out.append(row)
    return out


@st.composite
def weights(draw):
    N, M = draw(st.sampled_from(PATTERNS))
    n_out = draw(st.integers(1, 9))
    groups = draw(st.integers(1, 4))
    vals = draw(st.lists(st.integers(-3, 3), min_size=n_out * groups * M, max_size=n_out * groups * M))
    W = np.array(vals, dtype=np.int8).reshape(n_out, groups * M)
    tile = draw(st.integers(1, 5))
    return W, N, M, tile


@settings(max_examples=60, deadline=None)
@given(weights())
def test_row_rule_matches_enumeration(case):
    W, N, M, _ = case
    _, idx = oracle.compress(W, N, M)
    groups = W.shape[1] // M
    want = [[g * M + p for g in range(groups) for p in _best([abs(int(v)) for v in W[r, g * M:(g + 1) * M]], N)]
            for r in range(W.shape[0])]
    assert _positions(idx, groups, N, M) == want


@settings(max_examples=60, deadline=None)
@given(weights())
def test_tile_rule_matches_enumeration(case):
    W, N, M, V = case
    _, idx = oracle.compress_tile(W, N, M, tile=V)
    groups = W.shape[1] // M
    A = np.abs(W.astype(np.int64))
    want = []
    for r in range(W.shape[0]):
        rows = A[(r // V) * V:min((r // V) * V + V, W.shape[0])]
        want.append([g * M + p for g in range(groups) for p in _best(list(rows[:, g * M:(g + 1) * M].sum(0)), N)])
    assert _positions(idx, groups, N, M) == want


@settings(max_examples=40, deadline=None)
@given(weights(), st.integers(1, 6), st.integers(0, 2**31 - 1))
def test_masked_gemm_is_the_numpy_product(case, T, seed):
    W, N, M, V = case
    for values, idx in (oracle.compress(W, N, M), oracle.compress_tile(W, N, M, tile=V)):
        Wm = oracle.decompress(values, idx, W.shape[0], W.shape[1], N, M)
        kept = Wm != 0
        assert np.array_equal(Wm[kept], W[kept])                       # kept entries unchanged
        assert (np.count_nonzero(Wm.reshape(W.shape[0], -1, M), axis=2) <= N).all()
        X = np.random.default_rng(seed).integers(-128, 128, size=(T, W.shape[1])).astype(np.int8)
        assert np.array_equal(oracle.gemm(X, Wm), (X.astype(np.int64) @ Wm.astype(np.int64).T).astype(np.int32))
