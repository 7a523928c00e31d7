"""Tensor-parallel decode over head shards, with KV-head replication when there are fewer KV heads
than ranks.

Rank r of tp owns a consecutive run of Hq / tp query heads and either Hkv / tp whole KV heads (when
Hkv >= tp) or its own replica of the one KV head its query heads read (when Hkv < tp); the split is
``gqa_tp_shard`` of the C ABI (the kv-head-replication glossary entry of inferencex.semianalysis.com,
"Technical definition" and "Engineering details"; deepconcepts.dev Grouped-Query Attention, the
tensor-parallelism paragraphs of "Why nobody ships one kv head").  Attention itself needs no exchange:
each rank runs the ordinary decode on its shard (local group size q_count / kv_count), and the shards
are put back in head order by one all-gather of the outputs.  (A row-parallel output projection could
take the shards as they are; the all-gather is what a caller that wants the whole attention output
needs.)

Everything here is argument plumbing around the library: the shard arithmetic is the C ABI's, the
decode is the library's kernels, the gather is torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

from typing import Callable, NamedTuple


class TPShard(NamedTuple):
    q_first: int
    q_count: int
    kv_first: int
    kv_count: int


def tp_shard(Hq: int, Hkv: int, tp: int, rank: int) -> TPShard:
    """The query heads and KV heads rank ``rank`` of ``tp`` owns (gqa_tp_shard)."""
    from . import gqa_tp_shard

    return TPShard(*gqa_tp_shard(Hq, Hkv, tp, rank))


def take_shard(q, k_cache, v_cache, shard: TPShard):
    """What a rank holds of one layer: its query heads' rows of q [B, Hq, d] and its KV heads (or replica)
    of the caches [B, Tmax, Hkv, d], as contiguous tensors."""
    qs = q[:, shard.q_first:shard.q_first + shard.q_count].contiguous()
    ks = k_cache[:, :, shard.kv_first:shard.kv_first + shard.kv_count].contiguous()
    vs = v_cache[:, :, shard.kv_first:shard.kv_first + shard.kv_count].contiguous()
    return qs, ks, vs


def gather_heads(local, tp: int, group=None):
    """All-gather the ranks' outputs [B, q_count, d] and put them back in head order: rank r's run of
    heads is [r q_count, (r + 1) q_count), so the parts are concatenated in rank order."""
    import torch
    import torch.distributed as dist

    if tp == 1:
        return local
    parts = [torch.empty_like(local) for _ in range(tp)]
    dist.all_gather(parts, local.contiguous(), group=group)
    return torch.cat(parts, dim=1)


def tp_decode(q_shard, k_shard, v_shard, seqlens, scale: float, tp: int, group=None,
              decode: Callable | None = None):
    """One decode step of this rank's head shard, then the all-gather: returns the whole layer's
    attention output [B, Hq, d].  ``decode(q, k, v, seqlens, scale) -> out`` defaults to the library's
    ``gqa_decode``; a wrapper around ``gqa_decode_fp8`` serves an FP8 cache the same way."""
    if decode is None:
        from . import gqa_decode as decode
    local = decode(q_shard, k_shard, v_shard, seqlens, scale)
    return gather_heads(local, tp, group)
