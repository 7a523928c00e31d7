"""GPU parity of the MLA decode with absorbed weights against the fp64 oracle.

``gqa_mla_decode`` runs on the tensor cores and rounds the softmax weights to bf16 before the P.V
product, as the causal prefill does, so it is held to the prefill's derived gate (floor 2^-9
max|v|, v the latent rows that are the values).  ``gqa_mla_decode_cudacore`` keeps the weights in
fp32 and is held to the decode gate; at the full DeepSeek-V3-shaped size, where the oracle can
check only a few sequences in the time a test has, every output of the tensor-core kernel is also
compared with it.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import grouped_query_attention_02_b200 as gqa
from grouped_query_attention_02_b200 import inputs
from tests._tolerance import assert_close, compare

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(x, fn=None, **kw):
    fn = fn or gqa.gqa_mla_decode
    out = fn(x.q, x.kv_cache, x.seqlens, x.scale, **kw)
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    return out


def _ref(oracle_mod, x):
    return oracle_mod.mla_decode(x.q, x.kv_cache, x.seqlens.cpu(), x.d_c, x.scale)


def _vmax(x):
    """Largest |latent| over the rows inside the histories (the values the weights average)."""
    m = 0.0
    for b, t in enumerate(x.seqlens.cpu().tolist()):
        if t > 0:
            m = max(m, float(x.kv_cache[b, :t, :x.d_c].float().abs().max()))
    return m


def _check_tc(out, ref, x, **kw):
    return assert_close(out.double().cpu().numpy(), ref, kind="prefill", vmax=_vmax(x), **kw)


CASES = [
    (2, 20, 70, [70, 0]),            # a ragged head block and an empty history
    (1, 16, 600, [600]),             # one sequence: several pieces merged
    (3, 5, 300, [300, 33, 1]),       # fewer heads than a block, tile edges
    (2, 128, 1000, [1000, 517]),     # two head blocks
    (4, 16, 65, [32, 33, 64, 65]),   # partial tiles
    (3, 130, 257, [257, 128, 129]),  # a third, nearly empty head block; tile edges
]


@pytest.mark.parametrize("B,Hq,T,lens", CASES)
def test_mla_decode_small_cases(oracle_mod, B, Hq, T, lens):
    x = inputs.make_mla_decode(B, Hq, T, seqlens=lens, device=DEV, seed=B * 100 + Hq)
    ref = _ref(oracle_mod, x)
    out = _run(x)
    _check_tc(out, ref, x)
    for b, t in enumerate(lens):
        if t == 0:
            assert torch.all(out[b] == 0)


@pytest.mark.parametrize("B,Hq,T,lens", CASES)
def test_mla_decode_cudacore_small_cases(oracle_mod, B, Hq, T, lens):
    x = inputs.make_mla_decode(B, Hq, T, seqlens=lens, device=DEV, seed=B * 100 + Hq)
    out = _run(x, gqa.gqa_mla_decode_cudacore)
    assert_close(out.double().cpu().numpy(), _ref(oracle_mod, x))


def test_mla_decode_variable_lengths_many_pieces(oracle_mod):
    """Lengths from 1 to 16000 over 8 sequences: the planner cuts long histories into several
    pieces (merged by the combine), short ones stay whole, and last tiles are partial."""
    x = inputs.make_mla_decode(8, 64, 16000, device=DEV, seed=11, seqlen_range=(1, 16000))
    out = _run(x)
    ref = _ref(oracle_mod, x)
    _check_tc(out, ref, x)


def test_mla_decode_deepseek_shaped_full_vs_cudacore(oracle_mod):
    """The DeepSeek-V3-shaped decode the bench times (B=32, 128 heads, 512 + 64 wide rows, 8192 tokens):
    two sequences against the oracle, and every output against the CUDA-core path."""
    x = inputs.make_mla_decode(32, 128, 8192, device=DEV, seed=0)
    out = _run(x)
    for b in (0, 31):
        ref = oracle_mod.mla_decode(x.q[b:b + 1].cpu(), x.kv_cache[b:b + 1].cpu(), [8192], x.d_c, x.scale)
        vm = float(x.kv_cache[b, :, :x.d_c].float().abs().max())
        assert_close(out[b:b + 1].double().cpu().numpy(), ref, kind="prefill", vmax=vm)
    cc = _run(x, gqa.gqa_mla_decode_cudacore).double().cpu().numpy()
    tc = out.double().cpu().numpy()
    # both paths are within their gates of the exact result r: |tc - r| <= 2^-8|r| + 2^-9 vmax and
    # |cc - r| <= 2^-8|r| + 2^-10 max|r|; with |r| <= |cc| + |cc - r| their difference obeys the
    # bound below
    vmax = float(x.kv_cache[..., :x.d_c].float().abs().max())
    cmax = float(np.abs(cc).max())
    bound = 2.0 ** -7 * np.abs(cc) + 2.0 ** -9 * vmax + 2.0 ** -9 * cmax
    err = np.abs(tc - cc)
    assert not np.isnan(tc).any()
    assert np.all(err <= bound), float((err - bound).max())
    s = compare(tc, cc, kind="prefill", vmax=vmax)
    assert s["rel_normwise"] <= 2e-2, s


def test_mla_rows_past_the_history_are_never_read(oracle_mod):
    x = inputs.make_mla_decode(3, 16, 200, seqlens=[7, 150, 200], device=DEV, seed=6)
    for b, t in enumerate([7, 150, 200]):
        x.kv_cache[b, t:] = float("nan")
    out = _run(x)
    assert not torch.isnan(out).any()
    _check_tc(out, _ref(oracle_mod, x), x)


@pytest.mark.parametrize("fn", ["gqa_mla_decode", "gqa_mla_decode_cudacore"])
def test_mla_nan_inside_the_history_reaches_the_output(oracle_mod, fn):
    """A NaN anywhere in a cached row -- its RoPE key, or its latent, which is part of the key too --
    makes that token's score NaN for every head, so every output of that sequence is NaN; the other
    sequences are untouched."""
    x = inputs.make_mla_decode(3, 16, 300, seqlens=[300, 290, 300], device=DEV, seed=7)
    x.kv_cache[0, 100, 530] = float("nan")
    x.kv_cache[1, 3, 7] = float("nan")
    out = _run(x, getattr(gqa, fn)).double().cpu().numpy()
    ref = _ref(oracle_mod, x)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(out), nan)
    assert nan[0].all() and nan[1].all() and not nan[2].any()
    assert_close(out[2:], ref[2:], kind="prefill", vmax=float(x.kv_cache[2, :300, :x.d_c].float().abs().max()))


def test_mla_nan_inside_a_split_history(oracle_mod):
    """The same across pieces: a NaN in one piece of a long history makes the merged output NaN."""
    x = inputs.make_mla_decode(2, 64, 9000, seqlens=[9000, 9000], device=DEV, seed=12)
    x.kv_cache[0, 8500, 20] = float("nan")
    out = _run(x).double().cpu().numpy()
    assert np.isnan(out[0]).all() and not np.isnan(out[1]).any()


def test_mla_peaky_softmax(oracle_mod):
    x = inputs.make_mla_decode(2, 32, 900, seqlens=[900, 333], device=DEV, seed=8, q_gain=4.0)
    _check_tc(_run(x), _ref(oracle_mod, x), x, abs_bar=False)


def test_mla_deterministic_on_a_side_stream(oracle_mod):
    x = inputs.make_mla_decode(2, 16, 3000, seqlens=[3000, 1200], device=DEV, seed=9)
    a = _run(x)
    assert gqa.gqa_last_launch_count() == 3   # the plan, the decode and the combine of split histories
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = gqa.gqa_mla_decode(x.q, x.kv_cache, x.seqlens, x.scale, stream=s)
    s.synchronize()
    assert torch.equal(a, b)


def test_mla_decode_replays_in_a_cuda_graph(oracle_mod):
    """The planned MLA decode (planner, tensor-core kernel, combine) captured once in a CUDA graph and
    replayed, with new query rows in place between replays."""
    x = inputs.make_mla_decode(4, 64, 3000, device=DEV, seed=12, seqlen_range=(1, 3000))
    out = torch.empty((4, 64, x.d_c), dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gqa.gqa_mla_decode(x.q, x.kv_cache, x.seqlens, x.scale, out=out)   # sizes the workspace
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gqa.gqa_mla_decode(x.q, x.kv_cache, x.seqlens, x.scale, out=out)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    _check_tc(out, _ref(oracle_mod, x), x)
    x.q.copy_(inputs.make_mla_decode(4, 64, 3000, device=DEV, seed=13, seqlen_range=(1, 3000)).q)
    g.replay()
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    _check_tc(out, _ref(oracle_mod, x), x)
