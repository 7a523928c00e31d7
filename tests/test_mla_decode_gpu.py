"""GPU parity of the MLA decode with absorbed weights (gqa_mla_decode) against the fp64 oracle.

The oracle (``oracle.mla_decode``) is pinned to the MLA page's weight-absorption identity;
the kernel is checked with the same gates as the GQA decode (fp32 accumulation, bf16 output).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import grouped_query_attention_02_b200 as gqa
from grouped_query_attention_02_b200 import inputs
from tests._tolerance import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(x, **kw):
    out = gqa.gqa_mla_decode(x.q, x.kv_cache, x.seqlens, x.scale, **kw)
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    return out


def _ref(oracle_mod, x):
    return oracle_mod.mla_decode(x.q, x.kv_cache, x.seqlens.cpu(), x.d_c, x.scale)


@pytest.mark.parametrize("B,Hq,T,lens", [
    (2, 20, 70, [70, 0]),            # a ragged head block and an empty history
    (1, 16, 600, [600]),             # several token ranges merged
    (3, 5, 300, [300, 33, 1]),       # fewer heads than a block, tile edges
    (2, 128, 1000, [1000, 517]),     # all 128 heads
    (4, 16, 65, [32, 33, 64, 65]),   # tile edges
])
def test_mla_decode_small_cases(oracle_mod, B, Hq, T, lens):
    x = inputs.make_mla_decode(B, Hq, T, seqlens=lens, device=DEV, seed=B * 100 + Hq)
    out = _run(x)
    assert_close(out.double().cpu().numpy(), _ref(oracle_mod, x))
    for b, t in enumerate(lens):
        if t == 0:
            assert torch.all(out[b] == 0)


def test_mla_decode_deepseek_shaped_sampled(oracle_mod):
    """128 heads, 512 + 64 wide rows, 16 sequences of 8192 tokens; two sequences checked in full."""
    x = inputs.make_mla_decode(16, 128, 8192, device=DEV, seed=5)
    out = _run(x)
    for b in (0, 15):
        ref = oracle_mod.mla_decode(x.q[b:b + 1].cpu(), x.kv_cache[b:b + 1].cpu(), [8192], x.d_c, x.scale)
        assert_close(out[b:b + 1].double().cpu().numpy(), ref)


def test_mla_rows_past_the_history_are_never_read(oracle_mod):
    x = inputs.make_mla_decode(3, 16, 200, seqlens=[7, 150, 200], device=DEV, seed=6)
    for b, t in enumerate([7, 150, 200]):
        x.kv_cache[b, t:] = float("nan")
    out = _run(x)
    assert not torch.isnan(out).any()
    assert_close(out.double().cpu().numpy(), _ref(oracle_mod, x))


def test_mla_nan_inside_the_history_reaches_the_output(oracle_mod):
    """A NaN anywhere in a cached row -- its RoPE key, or its latent, which is part of the key too --
    makes that token's score NaN for every head, so every output of that sequence is NaN; the other
    sequences are untouched."""
    x = inputs.make_mla_decode(3, 16, 300, seqlens=[300, 290, 300], device=DEV, seed=7)
    x.kv_cache[0, 100, 530] = float("nan")
    x.kv_cache[1, 3, 7] = float("nan")
    out = _run(x).double().cpu().numpy()
    ref = _ref(oracle_mod, x)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(out), nan)
    assert nan[0].all() and nan[1].all() and not nan[2].any()
    assert_close(out[2:], ref[2:])


def test_mla_peaky_softmax(oracle_mod):
    x = inputs.make_mla_decode(2, 32, 900, seqlens=[900, 333], device=DEV, seed=8, q_gain=4.0)
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x), abs_bar=False)


def test_mla_deterministic_on_a_side_stream(oracle_mod):
    x = inputs.make_mla_decode(2, 16, 3000, seqlens=[3000, 1200], device=DEV, seed=9)
    a = _run(x)
    assert gqa.gqa_last_launch_count() == 2   # the decode and the combine of its token ranges
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = gqa.gqa_mla_decode(x.q, x.kv_cache, x.seqlens, x.scale, stream=s)
    s.synchronize()
    assert torch.equal(a, b)
