"""GPU parity of the decode path against the fp64 oracle, through the C ABI.

Small cases are compared element by element over every output; the full-size
workloads are compared on sampled sequences (every query head of each sampled
sequence), the oracle reading only those sequences' cached rows.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import grouped_query_attention_02_b200 as gqa
from grouped_query_attention_02_b200 import inputs, workloads
from tests._tolerance import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _oracle_rows(oracle_mod, x, bs):
    """Oracle outputs for sequences bs, one sequence at a time (copies only [0:T_b] rows)."""
    sl = x.seqlens.cpu().tolist()
    res = []
    for b in bs:
        T = max(1, sl[b])
        o = oracle_mod.decode(x.q[b:b + 1].cpu(), x.k_cache[b:b + 1, :T].cpu(), x.v_cache[b:b + 1, :T].cpu(),
                              [sl[b]], x.scale)
        res.append(o[0])
    return np.stack(res)


def _run(x, **kw):
    out = gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, **kw)
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    return out


def _check_all(oracle_mod, x, out):
    ref = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens.cpu(), x.scale)
    return assert_close(out.double().cpu().numpy(), ref)


# ---------------------------------------------------------------- the workloads


def test_tiny_decode_full(oracle_mod):
    w = workloads.TINY_DECODE
    x = inputs.make_decode(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device=DEV, seed=0)
    _check_all(oracle_mod, x, _run(x))


def test_qwen3_8b_shaped_decode_full(oracle_mod):
    w = workloads.QWEN3_8B_DECODE
    x = inputs.make_decode(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device=DEV, seed=0)
    _check_all(oracle_mod, x, _run(x))


@pytest.mark.parametrize("w", workloads.VARLEN_DECODE, ids=lambda w: f"Hkv{w.Hkv}")
def test_variable_length_decode_sampled(oracle_mod, w):
    x = inputs.make_decode(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device=DEV, seed=0, seqlen_range=w.seqlen_range)
    out = _run(x)
    sl = x.seqlens.cpu()
    bs = sorted({int(sl.argmin()), int(sl.argmax()), 0, 1, w.B // 2, w.B - 1})
    assert_close(out[bs].double().cpu().numpy(), _oracle_rows(oracle_mod, x, bs))


def test_extreme_grouping_decode_sampled(oracle_mod):
    w = workloads.EXTREME_GROUP_DECODE
    x = inputs.make_decode(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device=DEV, seed=0)
    out = _run(x)
    bs = [0, 7, 15]
    assert_close(out[bs].double().cpu().numpy(), _oracle_rows(oracle_mod, x, bs))


# ---------------------------------------------------------------- edges


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (6, 2), (8, 2), (32, 4), (32, 2), (32, 1), (71, 1)])
def test_group_sizes(oracle_mod, Hq, Hkv):
    x = inputs.make_decode(3, Hq, Hkv, 128, 300, seqlens=[300, 129, 17], device=DEV, seed=Hq * 10 + Hkv)
    _check_all(oracle_mod, x, _run(x))


def test_tile_edges_and_empty(oracle_mod):
    lens = [0, 1, 2, 63, 64, 65, 127, 128, 129, 1000, 1024, 1025]
    x = inputs.make_decode(len(lens), 8, 2, 128, 1025, seqlens=lens, device=DEV, seed=3)
    out = _run(x)
    assert torch.all(out[0] == 0)
    _check_all(oracle_mod, x, out)


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (24, 8), (32, 1)])
def test_short_caches_one_launch_more_units_than_ctas(oracle_mod, Hq, Hkv):
    """Caches of at most four 128-token tiles run as one launch over whole histories, dealt round-robin:
    here more (sequence, KV head) units than CTAs for the grouped shapes, lengths from 0 to 512."""
    B = 150
    lens = [(i * 37) % 513 for i in range(B)]
    x = inputs.make_decode(B, Hq, Hkv, 128, 512, seqlens=lens, device=DEV, seed=14 + Hkv)
    out = _run(x)
    assert gqa.gqa_last_launch_count() == 1
    for b, T in enumerate(lens):
        if T == 0:
            assert torch.all(out[b] == 0)
    _check_all(oracle_mod, x, out)


def test_split_boundaries(oracle_mod):
    # a long single sequence is split; lengths straddling the split chunk must merge exactly
    B, Hq, Hkv, Tmax = 2, 8, 2, 20000
    chunk, nsplit, _ = gqa.gqa_decode_plan(B, Hq, Hkv, 128, Tmax, torch.cuda.get_device_properties(0).multi_processor_count)
    assert nsplit > 1
    lens = [chunk + 1, min(Tmax, 2 * chunk - 1)]
    x = inputs.make_decode(B, Hq, Hkv, 128, Tmax, seqlens=lens, device=DEV, seed=4)
    _check_all(oracle_mod, x, _run(x))


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (32, 1)])
def test_many_pieces_per_history(oracle_mod, Hq, Hkv):
    # one sequence of 128 tiles on 148 SMs: the planner cuts it into the most pieces allowed (64, two tiles
    # each), so the merge runs well past the pieces it fetches together with the count
    x = inputs.make_decode(1, Hq, Hkv, 128, 16384, device=DEV, seed=70 + Hq)
    _check_all(oracle_mod, x, _run(x))


@pytest.mark.parametrize("B", [2500, 4200])
def test_large_batch_planned_by_one_warp(oracle_mod, B):
    # thousands of histories (78 or 131 per planner lane; past 4096 the planner re-reads lengths it does
    # not keep), some empty, some one tile, most split into pieces
    Hq, Hkv, Tmax = 8, 2, 640
    g = torch.Generator().manual_seed(90)
    lens = torch.randint(0, Tmax + 1, (B,), generator=g)
    lens[::97] = 0
    lens[5::89] = 1
    lens[7::83] = Tmax
    x = inputs.make_decode(B, Hq, Hkv, 128, Tmax, seqlens=lens.tolist(), device=DEV, seed=91)
    out = _run(x)
    sl = x.seqlens.cpu()
    bs = sorted({0, 1, 5, 7, 97, 1249, B - 1, int(sl.argmax()), int(sl.argmin())} | set(range(1200, 1216)) |
                set(range(min(B, 4090), min(B, 4102))))
    assert_close(out[bs].double().cpu().numpy(), _oracle_rows(oracle_mod, x, bs))


def test_nan_poisoned_padding_is_never_read(oracle_mod):
    lens = [5, 64, 100, 777]
    x = inputs.make_decode(4, 16, 4, 128, 800, seqlens=lens, device=DEV, seed=5, poison=True)
    out = _run(x)
    assert not torch.isnan(out).any()
    _check_all(oracle_mod, x, out)


@pytest.mark.parametrize("Hq,Hkv,T", [(8, 2, 300), (8, 2, 20000), (8, 8, 300), (8, 8, 20000), (71, 1, 3000)])
def test_nan_inside_the_history_reaches_the_output(oracle_mod, Hq, Hkv, T):
    """A NaN key makes its token's scores NaN for the whole group (all of their outputs NaN); a NaN value
    coordinate poisons that coordinate of the group's outputs, in one piece or across split pieces."""
    x = inputs.make_decode(2, Hq, Hkv, 128, T, seqlens=[T, T - 7], device=DEV, seed=21)
    g = Hq // Hkv
    x.k_cache[0, T // 3, Hkv - 1, 17] = float("nan")
    x.v_cache[1, T - 9, 0, 3] = float("nan")
    out = _run(x).double().cpu().numpy()
    ref = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens.cpu(), x.scale)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(out), nan)
    assert nan[0, (Hkv - 1) * g:].all() and nan[1, :g, 3].all() and int(nan.sum()) == g * 128 + g
    assert_close(np.where(nan, 0.0, out), np.where(nan, 0.0, ref))


@pytest.mark.parametrize("Hq,Hkv,tp", [(32, 8, 2), (32, 8, 8), (32, 2, 8), (8, 2, 4), (8, 1, 8)])
def test_tensor_parallel_shards_decoded_in_turn(oracle_mod, Hq, Hkv, tp):
    """Each tensor-parallel rank's shard (gqa_tp_shard: its query heads with its KV heads, or its replica
    of one) decoded in turn on this GPU -- the shards are independent, no rank waits on another -- and put
    back in head order: the unsharded decode of the oracle."""
    x = inputs.make_decode(3, Hq, Hkv, 128, 1500, seqlens=[1500, 700, 129], device=DEV, seed=51)
    whole = torch.empty_like(x.q)
    for r in range(tp):
        qf, qc, kf, kc = gqa.gqa_tp_shard(Hq, Hkv, tp, r)
        whole[:, qf:qf + qc] = gqa.gqa_decode(x.q[:, qf:qf + qc].contiguous(),
                                              x.k_cache[:, :, kf:kf + kc].contiguous(),
                                              x.v_cache[:, :, kf:kf + kc].contiguous(), x.seqlens, x.scale)
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    assert_close(whole.double().cpu().numpy(),
                 oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens.cpu(), x.scale))


def test_peaky_softmax(oracle_mod):
    x = inputs.make_decode(4, 32, 8, 128, 2048, seqlens=[2048, 1500, 33, 700], device=DEV, seed=6, q_gain=8.0)
    _check_all(oracle_mod, x, _run(x))


def test_lengths_outside_the_cache_are_clamped(oracle_mod):
    x = inputs.make_decode(2, 8, 2, 128, 128, seqlens=[128, 0], device=DEV, seed=7)
    out_ref = _run(x)
    x.seqlens = torch.tensor([128 + 50, -3], dtype=torch.int32, device=DEV)
    out = _run(x)
    assert torch.equal(out, out_ref)
    assert torch.all(out[1] == 0)


def test_non_default_stream_and_out_buffer(oracle_mod):
    x = inputs.make_decode(2, 8, 2, 128, 512, seqlens=[512, 300], device=DEV, seed=8)
    s = torch.cuda.Stream()
    out = torch.full_like(x.q, float("nan"))
    with torch.cuda.stream(s):
        gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, out=out, stream=s)
    s.synchronize()
    _check_all(oracle_mod, x, out)


def test_repeated_calls_are_deterministic():
    x = inputs.make_decode(8, 32, 8, 128, 4096, device=DEV, seed=9)
    a = _run(x).clone()
    b = _run(x)
    assert torch.equal(a, b)


# ---------------------------------------------------------------- expanded baseline


def test_expanded_baseline_matches_oracle(oracle_mod):
    x = inputs.make_decode(3, 32, 8, 128, 1500, seqlens=[1500, 999, 64], device=DEV, seed=10)
    out = gqa.gqa_decode_expanded(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    torch.cuda.synchronize()
    assert gqa.gqa_last_launch_count() >= 2
    _check_all(oracle_mod, x, out)


def test_expanded_copy_is_a_real_repeat():
    x = inputs.make_decode(2, 8, 2, 128, 100, seqlens=[100, 40], device=DEV, seed=11)
    k_rep = torch.zeros((2, 100, 8, 128), dtype=torch.bfloat16, device=DEV)
    v_rep = torch.zeros_like(k_rep)
    gqa.gqa_decode_expanded(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, k_rep=k_rep, v_rep=v_rep)
    torch.cuda.synchronize()
    for b, T in enumerate([100, 40]):
        assert torch.equal(k_rep[b, :T], x.k_cache[b, :T].repeat_interleave(4, dim=1))
        assert torch.equal(v_rep[b, :T], x.v_cache[b, :T].repeat_interleave(4, dim=1))
        assert torch.all(k_rep[b, T:] == 0)


# ---------------------------------------------------------------- failure detection


def test_bounded_wait_reports_timeout_and_context_survives(oracle_mod):
    gqa.gqa_selftest_wait_timeout(2000)
    assert gqa.gqa_get_last_device_status() == 6
    assert gqa.gqa_get_last_device_status() == 0          # read-and-clear
    x = inputs.make_decode(1, 8, 2, 128, 256, device=DEV, seed=12)
    _check_all(oracle_mod, x, _run(x))


def test_profile_events_bracket_the_decode_kernel():
    x = inputs.make_decode(16, 32, 8, 128, 4096, device=DEV, seed=13)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gqa.gqa_set_profile_events(e0, e1)
    try:
        _run(x)
    finally:
        gqa.gqa_set_profile_events(None, None)
    assert e0.elapsed_time(e1) > 0


# ---------------------------------------------------------------- CUDA graphs


@pytest.mark.parametrize("shape", [(1, 8, 2, 256, None), (4, 32, 8, 4096, [4096, 3000, 129, 1]), (3, 32, 1, 3000, None)],
                         ids=["one-launch", "planned-split", "mqa"])
def test_decode_replays_in_a_cuda_graph(oracle_mod, shape):
    """A decode call captured once in a CUDA graph and replayed: no allocation, host work or
    synchronisation inside the call (after a first call has sized the workspace), and the graph reads
    the live inputs at every replay."""
    B, Hq, Hkv, Tmax, lens = shape
    x = inputs.make_decode(B, Hq, Hkv, 128, Tmax, seqlens=lens, device=DEV, seed=60 + Hkv)
    out = torch.empty_like(x.q)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, out=out)   # sizes the workspace
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, out=out)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    _check_all(oracle_mod, x, out)
    # new query rows in place: the replay must see them
    x.q.copy_(inputs.make_decode(B, Hq, Hkv, 128, Tmax, seqlens=lens, device=DEV, seed=160 + Hkv).q)
    g.replay()
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    _check_all(oracle_mod, x, out)

