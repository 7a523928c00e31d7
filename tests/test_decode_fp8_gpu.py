"""GPU parity of the FP8 (E4M3) KV-cache decode against the fp64 oracle, through the C ABI.

The oracle widens each code from the E4M3 definition and multiplies by the
per-tensor scale; the kernel must match it to the same tolerance as the bf16
decode (its codes are widened exactly, the arithmetic is the same).
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


def _run(x, **kw):
    out = gqa.gqa_decode_fp8(x.q, x.k_cache, x.v_cache, x.seqlens, x.k_scale, x.v_scale, x.scale, **kw)
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    return out


def _ref(oracle_mod, x):
    return oracle_mod.decode_fp8(x.q, x.k_cache, x.v_cache, x.k_scale, x.v_scale, x.seqlens.cpu(), x.scale)


def _oracle_rows(oracle_mod, x, bs):
    sl = x.seqlens.cpu().tolist()
    res = []
    for b in bs:
        T = max(1, sl[b])
        o = oracle_mod.decode_fp8(x.q[b:b + 1].cpu(), x.k_cache[b:b + 1, :T].cpu(), x.v_cache[b:b + 1, :T].cpu(),
                                  x.k_scale, x.v_scale, [sl[b]], x.scale)
        res.append(o[0])
    return np.stack(res)


def test_tiny_fp8_decode_full(oracle_mod):
    w = workloads.TINY_DECODE
    x = inputs.make_decode_fp8(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device=DEV, seed=0)
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x))


def test_qwen3_8b_shaped_fp8_decode_sampled(oracle_mod):
    w = workloads.QWEN3_8B_DECODE
    x = inputs.make_decode_fp8(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device=DEV, seed=0)
    out = _run(x)
    bs = [0, 17, 48]
    assert_close(out[bs].double().cpu().numpy(), _oracle_rows(oracle_mod, x, bs))


@pytest.mark.parametrize("w", workloads.VARLEN_DECODE, ids=lambda w: f"Hkv{w.Hkv}")
def test_variable_length_fp8_decode_sampled(oracle_mod, w):
    x = inputs.make_decode_fp8(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device=DEV, seed=0, seqlen_range=w.seqlen_range)
    out = _run(x)
    sl = x.seqlens.cpu()
    bs = sorted({int(sl.argmin()), int(sl.argmax()), 0, w.B - 1})
    assert_close(out[bs].double().cpu().numpy(), _oracle_rows(oracle_mod, x, bs))


def test_extreme_grouping_fp8_decode_sampled(oracle_mod):
    w = workloads.EXTREME_GROUP_DECODE
    x = inputs.make_decode_fp8(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device=DEV, seed=0)
    out = _run(x)
    bs = [0, 15]
    assert_close(out[bs].double().cpu().numpy(), _oracle_rows(oracle_mod, x, bs))


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (6, 2), (8, 2), (16, 1), (32, 4), (24, 1), (32, 1)])
def test_fp8_group_sizes(oracle_mod, Hq, Hkv):
    x = inputs.make_decode_fp8(3, Hq, Hkv, 128, 300, seqlens=[300, 129, 17], device=DEV, seed=Hq * 10 + Hkv)
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x))


def test_fp8_tile_edges_and_empty(oracle_mod):
    lens = [0, 1, 2, 127, 128, 129, 255, 256, 257, 1000, 1025]
    x = inputs.make_decode_fp8(len(lens), 8, 2, 128, 1025, seqlens=lens, device=DEV, seed=3)
    out = _run(x)
    assert torch.all(out[0] == 0)
    assert_close(out.double().cpu().numpy(), _ref(oracle_mod, x))


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (32, 1)])
def test_fp8_short_caches_one_launch(oracle_mod, Hq, Hkv):
    # at most four tiles: one launch over whole histories, more units than CTAs, empty histories included
    B = 150
    lens = [(i * 41) % 513 for i in range(B)]
    x = inputs.make_decode_fp8(B, Hq, Hkv, 128, 512, seqlens=lens, device=DEV, seed=31 + Hkv)
    out = _run(x)
    assert gqa.gqa_last_launch_count() == 1
    assert torch.all(out[0] == 0)
    assert_close(out.double().cpu().numpy(), _ref(oracle_mod, x))


def test_fp8_long_history_split_and_merged(oracle_mod):
    x = inputs.make_decode_fp8(2, 8, 2, 128, 20000, seqlens=[20000, 9001], device=DEV, seed=4)
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x))


def test_fp8_nan_codes_past_the_history_are_never_read(oracle_mod):
    x = inputs.make_decode_fp8(4, 16, 4, 128, 800, seqlens=[5, 64, 100, 777], device=DEV, seed=5, poison=True)
    out = _run(x)
    assert not torch.isnan(out).any()
    assert_close(out.double().cpu().numpy(), _ref(oracle_mod, x))


@pytest.mark.parametrize("ks,vs", [(1.0, 1.0), (0.0021, 3.7), (-0.02, 0.5), (0.0, 1.0)])
def test_fp8_scales(oracle_mod, ks, vs):
    """Unit, small/large, negative and zero key scales (zero: a uniform softmax)."""
    x = inputs.make_decode_fp8(2, 8, 2, 128, 700, seqlens=[700, 300], device=DEV, seed=8, k_scale=ks, v_scale=vs)
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x))


@pytest.mark.parametrize("gain", [1e-30, 1e-6, 300.0])
def test_fp8_query_magnitudes(oracle_mod, gain):
    """Per-head power-of-two scaling of q keeps tiny and large queries exact in f16."""
    x = inputs.make_decode_fp8(2, 8, 2, 128, 500, seqlens=[500, 200], device=DEV, seed=9, q_gain=gain)
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x), abs_bar=gain < 100)


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (16, 1), (32, 1)])
def test_fp8_query_with_a_wide_range(oracle_mod, Hq, Hkv):
    # the scores are E4M3 products with the query split into two E4M3 terms per head: elements spread
    # over 2^0 .. 2^-24 of a head's largest (every bf16 exponent step the split handles differently:
    # exact, exact with a subnormal residual, rounded, flushed), with the largest element once per head
    x = inputs.make_decode_fp8(2, Hq, Hkv, 128, 700, seqlens=[700, 129], device=DEV, seed=31 + Hq)
    g = torch.Generator().manual_seed(32 + Hq)
    mag = torch.pow(2.0, -torch.randint(0, 25, (2, Hq, 128), generator=g).double())
    sign = torch.where(torch.rand((2, Hq, 128), generator=g) < 0.5, -1.0, 1.0).double()
    q = (mag * sign * 3.0).to(torch.bfloat16)
    q[:, :, 5] = 3.0   # the head's largest
    x = inputs.DecodeFp8Inputs(q.to(DEV), x.k_cache, x.v_cache, x.k_scale, x.v_scale, x.seqlens, x.scale)
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x))


def test_fp8_peaky_softmax(oracle_mod):
    x = inputs.make_decode_fp8(4, 32, 8, 128, 2048, seqlens=[2048, 1500, 33, 700], device=DEV, seed=6, q_gain=8.0)
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x), abs_bar=False)


def test_fp8_deterministic_and_on_a_side_stream(oracle_mod):
    x = inputs.make_decode_fp8(3, 32, 8, 128, 3000, seqlens=[3000, 10, 2222], device=DEV, seed=10)
    a = _run(x)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = gqa.gqa_decode_fp8(x.q, x.k_cache, x.v_cache, x.seqlens, x.k_scale, x.v_scale, x.scale, stream=s)
    s.synchronize()
    assert torch.equal(a, b)
    assert gqa.gqa_last_launch_count() == 3


def test_fp8_accepts_float8_tensors(oracle_mod):
    x = inputs.make_decode_fp8(1, 8, 2, 128, 256, device=DEV, seed=11)
    a = _run(x)
    b = gqa.gqa_decode_fp8(x.q, x.k_cache.view(torch.float8_e4m3fn), x.v_cache.view(torch.float8_e4m3fn),
                           x.seqlens, x.k_scale, x.v_scale, x.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def _e4m3_values():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double()


def test_fp8_every_value_code_reaches_the_output_exactly(oracle_mod):
    """One cached token per sequence: the output is v_scale times the widened value codes, so every one
    of the 256 codes (subnormals, both zeros and the two NaNs included) is checked to bf16 rounding."""
    x = inputs.make_decode_fp8(2, 2, 1, 128, 1, device=DEV, seed=12, v_scale=0.37)
    v = torch.arange(256, dtype=torch.int32).to(torch.uint8).reshape(2, 1, 1, 128)
    x.v_cache.copy_(v.to(DEV))
    out = _run(x).double().cpu().numpy()
    ref = _ref(oracle_mod, x)
    assert np.array_equal(np.isnan(out), np.isnan(ref)) and int(np.isnan(ref).sum()) == 2 * 2
    fin = ~np.isnan(ref)
    assert np.all(np.abs(out[fin] - ref[fin]) <= np.abs(ref[fin]) * 2.0 ** -8)


def test_fp8_every_key_code_moves_the_weights_as_its_value(oracle_mod):
    """Sequence b holds two tokens: key 0 is code b in coordinate 0 (zeros elsewhere), key 1 is zero; the
    values are +1 and -1, so the output is v_scale * tanh(s / 2) with s the first token's score.  The
    query is the power of two that puts |s| near 1 for that code, so each key code is checked through
    the scores to a few bf16 steps."""
    B = 256
    x = inputs.make_decode_fp8(B, 1, 1, 128, 2, device=DEV, seed=13, k_scale=1.0 / 64, v_scale=1.0)
    k = torch.zeros(B, 2, 1, 128, dtype=torch.uint8)
    k[:, 0, 0, 0] = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    v = torch.empty(B, 2, 1, 128, dtype=torch.uint8)
    v[:, 0] = 0x38   # +1.0
    v[:, 1] = 0xB8   # -1.0
    vals = _e4m3_values()
    q = torch.zeros(B, 1, 128, dtype=torch.float64)
    mag = (vals.abs() * x.k_scale * x.scale).clamp_min(1e-30)
    q[:, 0, 0] = torch.where(torch.isfinite(vals) & (vals != 0), torch.exp2(-torch.round(torch.log2(mag))), 1.0)
    x.k_cache.copy_(k.to(DEV))
    x.v_cache.copy_(v.to(DEV))
    x.q.copy_(q.to(torch.bfloat16).to(DEV))
    out = _run(x).double().cpu().numpy()
    ref = _ref(oracle_mod, x)
    assert np.array_equal(np.isnan(out), np.isnan(ref)) and int(np.isnan(ref[:, 0, 0]).sum()) == 2
    fin = ~np.isnan(ref)
    assert np.all(out[fin][np.abs(ref[fin]) == 0] == 0)
    assert np.all(np.abs(out[fin] - ref[fin]) <= np.abs(ref[fin]) * 2.0 ** -7 + 1e-30)


@pytest.mark.parametrize("frac_subnormal", [1.0, 0.5])
def test_fp8_subnormal_codes(oracle_mod, frac_subnormal):
    """Caches of E4M3 subnormals (exponent field 0), alone or mixed with normal codes, with scales that
    make them matter: the keys spread the scores over several units and the values set the output."""
    x = inputs.make_decode_fp8(3, 8, 2, 128, 400, seqlens=[400, 257, 31], device=DEV, seed=14,
                               k_scale=64.0, v_scale=64.0, q_gain=4.0)
    g = torch.Generator().manual_seed(15)
    for c in (x.k_cache, x.v_cache):
        sub = torch.randint(0, 8, c.shape, generator=g, dtype=torch.int32) | (torch.randint(0, 2, c.shape, generator=g, dtype=torch.int32) << 7)
        keep = torch.rand(c.shape, generator=g) >= frac_subnormal
        c.copy_(torch.where(keep, c.cpu().to(torch.int32), sub).to(torch.uint8).to(DEV))
    assert_close(_run(x).double().cpu().numpy(), _ref(oracle_mod, x))


def test_fp8_nan_codes_inside_the_history_propagate(oracle_mod):
    """A NaN key code turns its token's scores into NaN for every head of the group (all of their
    outputs NaN); a NaN value code poisons that coordinate of the group's outputs only, as in the oracle."""
    x = inputs.make_decode_fp8(2, 8, 2, 128, 300, seqlens=[300, 250], device=DEV, seed=16)
    x.k_cache[0, 5, 1, 17] = 0x7F
    x.v_cache[1, 200, 0, 3] = 0xFF
    out = _run(x).double().cpu().numpy()
    ref = _ref(oracle_mod, x)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(out), nan)
    assert nan[0, 4:].all() and nan[1, :4, 3].all() and int(nan.sum()) == 4 * 128 + 4
    assert_close(np.where(nan, 0.0, out), np.where(nan, 0.0, ref))


def test_fp8_rejects_groups_above_32():
    x = inputs.make_decode_fp8(1, 64, 1, 128, 128, device=DEV, seed=12)
    with pytest.raises(gqa.GQAError) as e:
        gqa.gqa_decode_fp8(x.q, x.k_cache, x.v_cache, x.seqlens, x.k_scale, x.v_scale, x.scale)
    assert e.value.status == 2
