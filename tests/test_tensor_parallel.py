"""Tensor-parallel head sharding (gqa_tp_shard) without a GPU.

Pinned to the pages: the kv-head-replication glossary entry (inferencex.semianalysis.com:
32 query heads and 2 KV heads at TP8 give each rank 4 query heads, and four ranks need
the same KV head) and the tensor-parallelism paragraphs of deepconcepts.dev
Grouped-Query Attention (partition when there are at least as many KV heads as ranks,
a replica per rank otherwise, max(1, Hkv / tp) KV heads per rank, and Qwen3-8B's cache
staying at 18 KiB per token per rank at TP8 whatever the KV-head count from 8 down to 1).
"""
from __future__ import annotations

import pytest

import grouped_query_attention_02_b200 as gqa

INVALID, UNSUPPORTED = 1, 2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from grouped_query_attention_02_b200 import build

    build.build()
    gqa.load()


def _plan(Hq, Hkv, tp):
    return [gqa.gqa_tp_shard(Hq, Hkv, tp, r) for r in range(tp)]


def test_replication_example_from_the_pages():
    plan = _plan(32, 2, 8)
    assert [qc for _, qc, _, _ in plan] == [4] * 8
    assert [qf for qf, _, _, _ in plan] == list(range(0, 32, 4))
    assert [(kf, kc) for _, _, kf, kc in plan] == [(0, 1)] * 4 + [(1, 1)] * 4


@pytest.mark.parametrize("Hq", [32, 64])
@pytest.mark.parametrize("Hkv", [1, 2, 4, 8, 16, 32])
@pytest.mark.parametrize("tp", [1, 2, 4, 8])
def test_every_head_once_and_each_rank_holds_its_groups(oracle_mod, Hq, Hkv, tp):
    plan = _plan(Hq, Hkv, tp)
    owned = []
    holders = {}
    for qf, qc, kf, kc in plan:
        assert kc == max(1, Hkv // tp)
        owned += list(range(qf, qf + qc))
        for h in range(qf, qf + qc):
            assert kf <= oracle_mod.kv_head(h, Hq, Hkv) < kf + kc
        for j in range(kf, kf + kc):
            holders[j] = holders.get(j, 0) + 1
    assert owned == list(range(Hq))
    assert sorted(holders) == list(range(Hkv))
    assert set(holders.values()) == {max(1, tp // Hkv)}
    # stored KV heads over all ranks: the replicas cost as much as tp distinct heads would
    assert sum(kc for _, _, _, kc in plan) == max(Hkv, tp)


def test_qwen3_8b_cache_per_rank_stays_at_18_kib(oracle_mod):
    for Hkv in (8, 4, 2, 1):
        for r in range(8):
            _, _, _, kc = gqa.gqa_tp_shard(32, Hkv, 8, r)
            assert oracle_mod.kv_bytes(36, 1, kc, 128, 2) == 18 * 1024


@pytest.mark.parametrize("Hq,Hkv,tp,status", [
    (71, 1, 2, UNSUPPORTED),     # Falcon-7B's 71 query heads do not split over 2 ranks
    (32, 8, 3, UNSUPPORTED),
    (48, 6, 4, UNSUPPORTED),     # more KV heads than ranks, but not a multiple
    (24, 3, 8, UNSUPPORTED),     # fewer KV heads than ranks, tp not a multiple of Hkv
    (8, 3, 2, INVALID),          # Hq not a multiple of Hkv
    (8, 2, 0, INVALID),
])
def test_unsupported_and_invalid_splits(Hq, Hkv, tp, status):
    with pytest.raises(gqa.GQAError) as e:
        gqa.gqa_tp_shard(Hq, Hkv, tp, 0)
    assert e.value.status == status


def test_rank_outside_the_group_is_rejected():
    for r in (-1, 4):
        with pytest.raises(gqa.GQAError) as e:
            gqa.gqa_tp_shard(8, 2, 4, r)
        assert e.value.status == INVALID
