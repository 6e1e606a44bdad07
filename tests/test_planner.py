"""The planner's rules (adaptive parallelism: kernel, token tile, k-splits)
checked on the CPU through nm_plan_for_shape, which runs the same planning code
as nm_plan_query with the resident-cluster capacities given instead of queried
from a GPU.  The capacities below are those of a 148-SM GPU running one CTA per
SM; the GPU tests check nm_plan_query itself."""
import itertools
import math

import pytest
import torch

import structured_sparse_gemm_compress_b200 as nm

SMS = 148
PAIR = (74, 74, 74)                        # CTA pairs at token tiles 224 / 192 / 128
STREAM = (148, 74, 48, 37, 28, 24, 21, 18)  # clusters of 1 .. 8 one-SM CTAs

FORCED = ("NMSPMM_FORCE_BN", "NMSPMM_FORCE_SPLITK", "NMSPMM_FORCE_XS", "NMSPMM_FORCE_GRID",
          "NMSPMM_FORCE_PAIR", "NMSPMM_SPLIT_GLOBAL", "NMSPMM_CSPLIT")


@pytest.fixture(autouse=True)
def _no_forced_plan(monkeypatch):
    for k in FORCED:
        monkeypatch.delenv(k, raising=False)


def plan(dtype, n_out, k, T, N=2, M=4, sms=SMS, pair=PAIR, stream=STREAM):
    return nm.nm_plan_for_shape(dtype, n_out, k, N, M, T, sms, pair, stream)


@pytest.mark.parametrize("dtype,K,n_out,T,want", [
    (torch.int8, 768, 768, 12608, 1),      # 6 channel tiles, 3 x 99 pair tiles of 128 tokens
    (torch.int8, 768, 2304, 12608, 1),
    (torch.int8, 768, 384, 12608, 0),      # 3 channel tiles: the last pair would compute a padding tile
    (torch.int8, 768, 576, 100352, 0),     # 5 channel tiles
    (torch.int8, 768, 192, 12608, 0),      # 99 pair tiles, fewer than the SMs
    (torch.int8, 768, 768, 6272, 0),       # 3 x 49 = 147 pair tiles < 148 SMs
    (torch.int8, 96, 768, 100352, 0),      # under 192 bytes of X per token
    (torch.int8, 192, 768, 100352, 1),     # exactly 192 bytes
    (torch.int8, 3072, 384, 12608, 1),     # >= 2 KB of X per token: pair whatever the tile count
    (torch.float16, 768, 768, 6304, 1),    # 1536 bytes per token, 3 x 50 pair tiles
    (torch.float16, 1024, 1024, 6304, 1),  # 2 KB per token
    (torch.bfloat16, 96, 768, 12608, 1),   # 192 bytes per token
])
def test_pair_rule(dtype, K, n_out, T, want):
    assert plan(dtype, n_out, K, T)["pair"] == want


def test_pair_rule_follows_the_sm_count():
    # 147 pair tiles of 128 tokens: enough on a GPU of 147 SMs, not on one of 148
    assert plan(torch.int8, 768, 768, 6272, sms=148)["pair"] == 0
    assert plan(torch.int8, 768, 768, 6272, sms=147)["pair"] == 1


@pytest.mark.parametrize("n_out,K,bn", [(2304, 768, 224), (768, 768, 192), (3072, 768, 192), (768, 3072, 192)])
def test_pair_token_tile_minimises_rounds_times_tile_cost(n_out, K, bn):
    """ViT-B at T = 12608: the pair's token tile minimises rounds x (BN + 48)."""
    p = plan(torch.int8, n_out, K, 12608)
    assert p["pair"] == 1 and p["bn"] == bn and p["splits"] == 1 and p["cluster"] == 0
    pairs = math.ceil(math.ceil(n_out / 128) / 2)
    costs = {b: math.ceil(pairs * math.ceil(12608 / b) / 74) * (b + 48) for b in (224, 192, 128)}
    assert bn == min(costs, key=lambda b: (costs[b], -b))
    assert p["units"] == pairs * math.ceil(12608 / bn) and p["grid"] == min(p["units"], 74)


def test_pair_tile_that_cannot_run_is_skipped():
    # no room for 224-token pairs: the next best tile is taken
    p = plan(torch.int8, 2304, 768, 12608, pair=(0, 74, 74))
    assert p["pair"] == 1 and p["bn"] != 224
    # no pair fits at all: the one-SM kernel
    assert plan(torch.int8, 2304, 768, 12608, pair=(0, 0, 0))["pair"] == 0


@pytest.mark.parametrize("T", [16, 64])
def test_long_k_at_few_tokens_splits_on_chip(T):
    p = plan(torch.int8, 768, 3072, T)
    assert p["pair"] == 0 and p["splits"] > 1 and p["cluster"] == 1
    assert p["grid"] == p["units"] == math.ceil(768 / 128) * math.ceil(T / p["bn"]) * p["splits"]


@pytest.mark.parametrize("T", [16, 64, 197])
def test_three_k_block_layers_never_split(T):
    for n_out in (768, 2304, 3072):
        assert plan(torch.int8, n_out, 768, T)["splits"] == 1


def test_no_cluster_capacity_no_on_chip_split():
    p = plan(torch.int8, 768, 3072, 16, stream=(148, 0, 0, 0, 0, 0, 0, 0))
    assert p["splits"] == 1 and p["cluster"] == 0


def test_large_token_counts_never_split():
    for n_out, K in ((768, 768), (2304, 768), (3072, 768), (768, 3072)):
        assert plan(torch.int8, n_out, K, 12608)["splits"] == 1


def test_forced_overrides(monkeypatch):
    monkeypatch.setenv("NMSPMM_FORCE_PAIR", "0")
    assert plan(torch.int8, 2304, 768, 12608)["pair"] == 0
    monkeypatch.setenv("NMSPMM_FORCE_PAIR", "1")
    assert plan(torch.int8, 384, 768, 12608)["pair"] == 1        # forced onto an odd tile count
    monkeypatch.delenv("NMSPMM_FORCE_PAIR")
    monkeypatch.setenv("NMSPMM_FORCE_BN", "128")
    assert plan(torch.int8, 2304, 768, 12608)["bn"] == 128
    monkeypatch.delenv("NMSPMM_FORCE_BN")
    monkeypatch.setenv("NMSPMM_FORCE_SPLITK", "3")
    p = plan(torch.int8, 768, 3072, 300)
    assert p["pair"] == 0 and p["splits"] == 3 and p["cluster"] == 1
    monkeypatch.setenv("NMSPMM_SPLIT_GLOBAL", "1")
    assert plan(torch.int8, 768, 3072, 300)["cluster"] == 0     # the workspace reduction
    monkeypatch.delenv("NMSPMM_FORCE_SPLITK")
    monkeypatch.delenv("NMSPMM_SPLIT_GLOBAL")
    monkeypatch.setenv("NMSPMM_FORCE_GRID", "16")                # 16 persistent CTAs: 16 pair tiles suffice
    p = plan(torch.int8, 256, 768, 2000)
    assert p["pair"] == 1 and p["grid"] <= 8


def test_rejections():
    with pytest.raises(nm.NMError) as e:
        plan(torch.int8, 768, 768, 100, N=3, M=4)
    assert e.value.status == nm.NM_ERR_UNSUPPORTED
    for kw in ({"T": 0}, {"k": 770}, {"sms": 0}):
        args = dict(dtype=torch.int8, n_out=768, k=768, T=100)
        args.update(kw)
        with pytest.raises(nm.NMError) as e:
            plan(**args)
        assert e.value.status == nm.NM_ERR_INVALID


@pytest.mark.parametrize("dtype", [torch.int8, torch.float16])
def test_plan_invariants_over_shapes(dtype):
    """Whatever the shape: every unit is one (tile, split); the grid never
    exceeds the units or the resident capacity; splits own >= 1 k-block each."""
    kb_elems = 256 if dtype == torch.int8 else 128
    for (n_out, K, T), (N, M) in itertools.product(
            itertools.product((96, 200, 384, 768, 2304), (96, 256, 768, 3072), (1, 16, 197, 1000, 12608, 50432)),
            ((2, 4), (4, 8), (4, 4))):
        p = plan(dtype, n_out, K, T, N=N, M=M)
        n_ct, n_kb = math.ceil(n_out / 128), math.ceil(K / kb_elems)
        assert 1 <= p["splits"] <= n_kb
        if p["pair"]:
            assert p["bn"] in (224, 192, 128) and p["splits"] == 1 and p["cluster"] == 0
            assert p["units"] == math.ceil(n_ct / 2) * math.ceil(T / p["bn"])
            assert 1 <= p["grid"] <= min(p["units"], 74)
        else:
            assert p["bn"] in (32, 64, 128, 192)
            assert p["units"] == n_ct * math.ceil(T / p["bn"]) * p["splits"]
            if p["cluster"]:
                assert 2 <= p["splits"] <= 8 and p["grid"] == p["units"]
            else:
                assert 1 <= p["grid"] <= min(p["units"], SMS)
