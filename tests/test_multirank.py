"""Multi-rank host logic on CPU: two gloo ranks, as bench.py --gpus 2 would run them.

The decode shards by sequence with no exchange inside attention, so each rank
decodes its own sequences.  Checked here without a GPU:
* each rank's seeded inputs are what a single process would draw for that rank;
* concatenating the ranks' (oracle) outputs equals decoding the concatenated
  batch in one place: sharding by sequence needs no collective on the data path;
* the step time reported is the maximum over ranks and the value is all ranks'
  bytes over that time (bench.aggregate);
* tensor-parallel head sharding (tp.py over gqa_tp_shard, the rank logic of
  bench.py --tp): each rank decodes its own query heads against its KV heads, or
  its replica of one, and the all-gather puts the outputs back in head order,
  equal to the unsharded decode -- with KV heads partitioned (2 and 4 ranks, MHA
  included) and replicated (4 ranks).
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from grouped_query_attention_02_b200 import inputs

        per_rank = 3
        x = inputs.make_decode(per_rank, 8, 2, 16, 24, seqlens=[24, 9, 1], device="cpu", seed=bench.rank_seed(rank))
        out = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, nthreads=1)
        # each rank's "step time"; the job's time is the slowest rank's
        my_ms = 1.0 + rank
        t = torch.tensor([my_ms], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        gathered = [torch.zeros_like(torch.from_numpy(out)) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(out))
        if rank == 0:
            np.save(os.path.join(out_dir, "gathered.npy"), torch.cat(gathered).numpy())
            np.save(os.path.join(out_dir, "tmax.npy"), t.numpy())
            np.save(os.path.join(out_dir, "shards.npy"),
                    np.array([bench.shard_of(r, world, per_rank) for r in range(world)]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_by_sequence(tmp_path):
    import bench
    import oracle
    from grouped_query_attention_02_b200 import inputs

    oracle.build()
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    gathered = np.load(tmp_path / "gathered.npy")
    assert float(np.load(tmp_path / "tmax.npy")[0]) == 2.0
    shards = np.load(tmp_path / "shards.npy")
    assert shards.tolist() == [[0, 1, 2], [3, 4, 5]]
    # the same batch decoded in one place
    xs = [inputs.make_decode(3, 8, 2, 16, 24, seqlens=[24, 9, 1], device="cpu", seed=bench.rank_seed(r))
          for r in range(world)]
    q = torch.cat([x.q for x in xs])
    k = torch.cat([x.k_cache for x in xs])
    v = torch.cat([x.v_cache for x in xs])
    sl = torch.cat([x.seqlens for x in xs])
    whole = oracle.decode(q, k, v, sl, xs[0].scale, nthreads=1)
    np.testing.assert_array_equal(gathered, whole)
    # ranks draw different data
    assert not torch.equal(xs[0].k_cache, xs[1].k_cache)


def test_aggregate_uses_the_slowest_rank():
    import bench

    v, t = bench.aggregate([10.0, 10.0, 10.0], [1.0, 2.0, 1.5])
    assert t == 2.0 and v == 15.0
    assert bench.unique_kv_bytes([8192] * 49, 8, 128) == 1644167168      # the Qwen3-8B-shaped cache
    assert bench.prefill_causal_flops(4, 8192, 32, 128) == 2199291691008     # 2.199 TFLOP causal
    assert bench.decode_flops([8192], 32, 128) == 4 * 36 * 32 * 128 * 8192 // 36   # one layer of the 4.83 GFLOP figure


def _tp_worker(rank, world, port, out_dir, Hq, Hkv):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from grouped_query_attention_02_b200 import inputs, tp

        # the rank logic of bench.py --tp: every rank draws the same layer, keeps only its shard, decodes
        # it and all-gathers the outputs in head order (the CPU oracle stands in for the rank's GPU decode)
        x = inputs.make_decode(2, Hq, Hkv, 16, 20, seqlens=[20, 7], device="cpu", seed=41)
        shard = tp.tp_shard(Hq, Hkv, world, rank)
        qs, ks, vs = tp.take_shard(x.q, x.k_cache, x.v_cache, shard)
        assert ks.shape[2] == shard.kv_count and qs.shape[1] == Hq // world

        def cpu_decode(q, k, v, seqlens, scale):
            return torch.from_numpy(oracle.decode(q, k, v, seqlens, scale, nthreads=1))

        whole = tp.tp_decode(qs, ks, vs, x.seqlens, x.scale, world, decode=cpu_decode)
        if rank == 0:
            np.save(os.path.join(out_dir, "tp.npy"), whole.numpy())
            np.save(os.path.join(out_dir, "shards.npy"),
                    np.array([tuple(tp.tp_shard(Hq, Hkv, world, r)) for r in range(world)]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,Hq,Hkv", [(2, 8, 2), (4, 8, 2), (4, 8, 1), (4, 16, 8), (2, 8, 8)])
def test_tensor_parallel_shards_reassemble_the_decode(tmp_path, world, Hq, Hkv):
    import oracle
    from grouped_query_attention_02_b200 import build, inputs

    oracle.build()
    build.build()
    port = _free_port()
    mp.start_processes(_tp_worker, args=(world, port, str(tmp_path), Hq, Hkv), nprocs=world, start_method="spawn")
    got = np.load(tmp_path / "tp.npy")
    x = inputs.make_decode(2, Hq, Hkv, 16, 20, seqlens=[20, 7], device="cpu", seed=41)
    np.testing.assert_array_equal(got, oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, nthreads=1))
    shards = np.load(tmp_path / "shards.npy")
    # every query head owned once, in rank order; replicas when there are fewer KV heads than ranks
    assert shards[:, 0].tolist() == list(range(0, Hq, Hq // world))
    assert (shards[:, 3] == max(1, Hkv // world)).all()

