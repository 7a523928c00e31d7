"""Pins for the fp64 oracle: each check ties it to something other than itself.

* golden values printed on the pages (tests/golden/, each line cited);
* closed forms (the two-query example, one cached token, a zero query);
* library routines for special cases (torch scaled_dot_product_attention in
  fp64 for the MHA endpoint and for causal prefill, torch's own bf16 -> fp64
  conversion, torch.repeat_interleave for the expanded form);
* a grouped, copy-free restatement (queries of a group as extra rows against
  one shared KV head) that must agree with the oracle's explicit repeat;
* brute force in plain Python on tiny shapes with distinct per-head inputs;
* invariants (swapping two KV heads together with their query groups swaps
  the outputs group by group).
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import torch

from grouped_query_attention_02_b200 import inputs
from tests._tolerance import compare

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln


# ---------------------------------------------------------------- mapping


def test_mapping_matches_pages(oracle_mod):
    n = 0
    for ln in _lines("mapping.txt"):
        head, rest = ln.split(":")
        Hq, Hkv = map(int, head.split())
        expect = [int(x) for x in rest.split()[:Hq]]
        assert [oracle_mod.kv_head(h, Hq, Hkv) for h in range(Hq)] == expect
        n += 1
    assert n == 2


def test_mapping_endpoints_and_irregular(oracle_mod):
    assert [oracle_mod.kv_head(h, 12, 12) for h in range(12)] == list(range(12))  # MHA
    assert [oracle_mod.kv_head(h, 71, 1) for h in range(71)] == [0] * 71          # MQA, 71 heads
    assert oracle_mod.kv_head(0, 6, 4) == -1      # 6 query heads cannot split into 4 groups
    assert oracle_mod.kv_head(8, 8, 2) == -1      # out of range
    assert oracle_mod.kv_head(-1, 8, 2) == -1


# ---------------------------------------------------------------- byte model


def test_kv_bytes_match_pages(oracle_mod):
    n = 0
    for ln in _lines("kv_bytes.txt"):
        f = ln.split()
        L, T, H, d, b, expect = (int(x) for x in f[:6])
        assert oracle_mod.kv_bytes(L, T, H, d, b) == expect, ln
        n += 1
    assert n == 9


def test_kv_bytes_ratios(oracle_mod):
    # two-head GQA stores a quarter of eight-head MHA's raw cache; query heads never enter
    assert 4 * oracle_mod.kv_bytes(32, 4096, 2, 128, 2) == oracle_mod.kv_bytes(32, 4096, 8, 128, 2)
    # an 8k-token request of the 36-layer, 8-KV-head config: 1.125 GiB (the page rounds to 1.13)
    assert oracle_mod.kv_bytes(36, 8192, 8, 128, 2) == 1.125 * 2 ** 30
    assert oracle_mod.kv_bytes(32, 1, 32, 128, 2) == 4 * oracle_mod.kv_bytes(32, 1, 8, 128, 2) == 512 * 1024


def test_capacity_exercise(oracle_mod):
    for ln in _lines("capacity.txt"):
        L, H, d, w, expect = ln.split()
        free = (80 - float(w) - 4) * 2 ** 30
        per_request = oracle_mod.kv_bytes(int(L), 4096, int(H), int(d), 2)
        assert int(free // per_request) == int(expect)


# ---------------------------------------------------------------- bf16


def test_bf16_conversion_exhaustive(oracle_mod):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle_mod.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# ---------------------------------------------------------------- closed forms


def _bf(x):
    return torch.tensor(x, dtype=torch.float64).to(torch.bfloat16)


def test_two_query_example(oracle_mod):
    keys, values, queries = [], [], []
    for ln in _lines("two_query.txt"):
        f = ln.split()
        {"key": keys, "value": values, "query": queries}[f[0]].append([float(x) for x in f[1:]])
    d = 2
    q = _bf([queries])                       # [1, 2 heads, 2]
    k = _bf([[[kk] for kk in keys]])         # [1, T=2, 1 kv head, 2]
    v = _bf([[[vv] for vv in values]])
    out = oracle_mod.decode(q, k, v, [2], 1.0 / math.sqrt(d))
    a, b = out[0, 0, 0], out[0, 1, 0]
    c = math.exp(-1.0 / math.sqrt(2.0))
    assert a == pytest.approx((10 + 20 * c) / (1 + c), rel=1e-14)
    assert b == pytest.approx((10 * c + 20) / (1 + c), rel=1e-14)
    assert (round(a, 6), round(b, 6)) == (13.302385, 16.697615)
    assert not math.isclose(a, b)            # shared K/V, distinct queries, distinct outputs
    assert a + b == pytest.approx(30.0, rel=1e-14)   # mirror symmetry of the example
    assert out[0, 0, 1] == 0.0 and out[0, 1, 1] == 0.0


def test_single_cached_token_returns_its_value_row(oracle_mod):
    x = inputs.make_decode(2, 8, 2, 16, 5, seqlens=[1, 1], seed=11)
    out = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    v = x.v_cache.double().numpy()
    for h in range(8):
        for b in range(2):
            assert np.array_equal(out[b, h], v[b, 0, h // 4])


def test_zero_query_averages_values(oracle_mod):
    x = inputs.make_decode(2, 6, 2, 16, 7, seqlens=[7, 3], seed=5)
    q0 = torch.zeros_like(x.q)
    out = oracle_mod.decode(q0, x.k_cache, x.v_cache, x.seqlens, x.scale)
    v = x.v_cache.double().numpy()
    for b, T in enumerate([7, 3]):
        for h in range(6):
            np.testing.assert_allclose(out[b, h], v[b, :T, h // 3].mean(axis=0), rtol=0, atol=1e-14)


def test_empty_history_gives_zero(oracle_mod):
    x = inputs.make_decode(2, 4, 2, 16, 4, seqlens=[0, 4], seed=2)
    out = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert np.all(out[0] == 0.0)
    assert np.any(out[1] != 0.0)


def test_rejects_irregular_or_bad_lengths(oracle_mod):
    x = inputs.make_decode(1, 6, 2, 16, 4, seed=1)
    with pytest.raises(ValueError):
        oracle_mod.decode(x.q, x.k_cache[:, :, :1].expand(1, 4, 4, 16).contiguous(), x.v_cache[:, :, :1]
                          .expand(1, 4, 4, 16).contiguous(), x.seqlens, x.scale)
    with pytest.raises(ValueError):
        oracle_mod.decode(x.q, x.k_cache, x.v_cache, [5], x.scale)


# ---------------------------------------------------------------- library routines


def _sdpa(q, k, v, scale, causal=False):
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale, is_causal=causal)


def test_mha_endpoint_equals_library_sdpa(oracle_mod):
    x = inputs.make_decode(2, 4, 4, 16, 9, seqlens=[9, 5], seed=21)
    out = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    for b, T in enumerate([9, 5]):
        q = x.q[b].double()[:, None, :]                     # [H,1,d]
        k = x.k_cache[b, :T].double().transpose(0, 1)       # [H,T,d]
        v = x.v_cache[b, :T].double().transpose(0, 1)
        ref = _sdpa(q, k, v, x.scale)[:, 0, :].numpy()
        np.testing.assert_allclose(out[b], ref, rtol=1e-12, atol=1e-13)


def test_mqa_endpoint_equals_library_sdpa(oracle_mod):
    x = inputs.make_decode(2, 6, 1, 16, 8, seqlens=[8, 2], seed=22)
    out = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    for b, T in enumerate([8, 2]):
        q = x.q[b].double()[:, None, :]
        k = x.k_cache[b, :T, 0].double()[None].expand(6, T, 16)
        v = x.v_cache[b, :T, 0].double()[None].expand(6, T, 16)
        np.testing.assert_allclose(out[b], _sdpa(q, k, v, x.scale)[:, 0, :].numpy(), rtol=1e-12, atol=1e-13)


def test_prefill_mha_equals_library_causal_sdpa(oracle_mod):
    x = inputs.make_prefill(2, 9, 4, 4, 16, seed=23)
    out = oracle_mod.prefill_causal(x.q, x.k, x.v, x.scale)
    ref = _sdpa(x.q.double().transpose(1, 2), x.k.double().transpose(1, 2), x.v.double().transpose(1, 2),
                x.scale, causal=True).transpose(1, 2).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_prefill_grouped_equals_expanded_tiny(oracle_mod):
    """The page's equivalence case: B=2, T=9, 12 query heads, 3 KV heads, d=16, causal."""
    B, T, Hq, Hkv, d = 2, 9, 12, 3, 16
    rep = Hq // Hkv
    x = inputs.make_prefill(B, T, Hq, Hkv, d, seed=24)
    gqa = oracle_mod.prefill_causal(x.q, x.k, x.v, x.scale)
    # expanded: physically repeat K/V along the head axis with the library routine, then MHA
    k_rep = x.k.repeat_interleave(rep, dim=2).contiguous()
    v_rep = x.v.repeat_interleave(rep, dim=2).contiguous()
    mha = oracle_mod.prefill_causal(x.q, k_rep, v_rep, x.scale)
    np.testing.assert_array_equal(gqa, mha)
    # grouped without copies: a group's rep query heads become rep*T extra rows against one KV head
    q = x.q.double()                     # [B,T,Hq,d]
    k = x.k.double()
    v = x.v.double()
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    for j in range(Hkv):
        qg = q[:, :, j * rep:(j + 1) * rep, :].permute(0, 2, 1, 3).reshape(B, rep * T, d)
        s = (qg @ k[:, :, j, :].transpose(1, 2)) * x.scale             # [B, rep*T, T]
        s = s.view(B, rep, T, T).masked_fill(~causal, float("-inf"))
        o = torch.softmax(s, dim=-1).reshape(B, rep * T, T) @ v[:, :, j, :]
        o = o.view(B, rep, T, d).permute(0, 2, 1, 3).numpy()
        np.testing.assert_allclose(gqa[:, :, j * rep:(j + 1) * rep, :], o, rtol=1e-12, atol=1e-13)


def test_prefill_row_subset_matches_full(oracle_mod):
    x = inputs.make_prefill(2, 11, 6, 2, 16, seed=25)
    full = oracle_mod.prefill_causal(x.q, x.k, x.v, x.scale)
    rows = [(1, 5, 10), (0, 0, 0), (1, 2, 3), (0, 5, 7), (1, 5, 0)]
    sub = oracle_mod.prefill_causal(x.q, x.k, x.v, x.scale, rows=rows)
    for i, (b, h, r) in enumerate(rows):
        np.testing.assert_array_equal(sub[i], full[b, r, h])


# ---------------------------------------------------------------- brute force


def _brute_decode(q, k, v, seqlens, scale):
    """Plain-Python loops over flat lists; mapping written as integer division."""
    B, Hq, d = len(q), len(q[0]), len(q[0][0])
    Hkv = len(k[0][0])
    out = [[[0.0] * d for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            kv = h * Hkv // Hq
            T = seqlens[b]
            if T == 0:
                continue
            s = [scale * sum(q[b][h][j] * k[b][t][kv][j] for j in range(d)) for t in range(T)]
            w = [math.exp(x) for x in s]        # inputs are small: no max shift needed
            z = math.fsum(w)
            for j in range(d):
                out[b][h][j] = math.fsum(w[t] * v[b][t][kv][j] for t in range(T)) / z
    return out


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 1), (6, 2), (8, 2), (12, 3), (71, 1)])
@pytest.mark.parametrize("d", [2, 16])
def test_brute_force_decode(oracle_mod, Hq, Hkv, d):
    seqlens = [9, 1, 3, 2, 0]
    x = inputs.make_decode(5, Hq, Hkv, d, 9, seqlens=seqlens, seed=100 + Hq + d)
    got = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    ref = _brute_decode(x.q.double().tolist(), x.k_cache.double().tolist(), x.v_cache.double().tolist(),
                        seqlens, x.scale)
    np.testing.assert_allclose(got, np.array(ref), rtol=1e-12, atol=1e-13)


def test_brute_force_prefill(oracle_mod):
    B, S, Hq, Hkv, d = 2, 5, 6, 2, 4
    x = inputs.make_prefill(B, S, Hq, Hkv, d, seed=31)
    got = oracle_mod.prefill_causal(x.q, x.k, x.v, x.scale)
    q, k, v = x.q.double().tolist(), x.k.double().tolist(), x.v.double().tolist()
    for b in range(B):
        for r in range(S):
            for h in range(Hq):
                kv = h // (Hq // Hkv)
                w = [math.exp(x.scale * sum(q[b][r][h][j] * k[b][t][kv][j] for j in range(d)))
                     for t in range(r + 1)]
                z = math.fsum(w)
                for j in range(d):
                    ref = math.fsum(w[t] * v[b][t][kv][j] for t in range(r + 1)) / z
                    assert got[b, r, h, j] == pytest.approx(ref, rel=1e-12, abs=1e-13)


# ---------------------------------------------------------------- invariants


def test_swapping_kv_heads_with_their_groups_swaps_outputs(oracle_mod):
    B, Hq, Hkv, d, T = 2, 8, 2, 16, 6
    x = inputs.make_decode(B, Hq, Hkv, d, T, seed=41)
    base = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    g = Hq // Hkv
    perm_kv = [1, 0]
    perm_q = [perm_kv[h // g] * g + h % g for h in range(Hq)]
    out = oracle_mod.decode(x.q[:, perm_q].contiguous(), x.k_cache[:, :, perm_kv].contiguous(),
                            x.v_cache[:, :, perm_kv].contiguous(), x.seqlens, x.scale)
    np.testing.assert_array_equal(out, base[:, perm_q])
    # swapping only the KV heads must change the outputs (the mapping is not symmetric)
    out2 = oracle_mod.decode(x.q, x.k_cache[:, :, perm_kv].contiguous(), x.v_cache[:, :, perm_kv].contiguous(),
                             x.seqlens, x.scale)
    assert not np.allclose(out2, base)


def test_distinct_queries_in_a_group_give_distinct_outputs(oracle_mod):
    x = inputs.make_decode(1, 8, 2, 16, 32, seed=42)
    out = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    for h in range(1, 4):
        assert not np.allclose(out[0, 0], out[0, h])


def test_tight_tolerance_sees_one_dropped_token(oracle_mod):
    """At the tiny decode shape, an off-by-one in the cached length breaks the tight gate."""
    x = inputs.make_decode(1, 8, 2, 128, 256, seed=0)
    full = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    short = oracle_mod.decode(x.q, x.k_cache, x.v_cache, [255], x.scale)
    assert compare(short, full)["tight_violations"] > 0
    assert compare(full, full)["tight_violations"] == 0


# ---------------------------------------------------------------- FP8 (E4M3) KV cache


def _e4m3_f64(codes):
    """torch's own E4M3 -> float64 conversion (a library routine, independent of the oracle)."""
    t = torch.as_tensor(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_e4m3_conversion_exhaustive(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    got = oracle_mod.e4m3_to_f64(codes)
    ref = _e4m3_f64(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))   # 0x80 is -0


def test_e4m3_format_constants(oracle_mod):
    """Fixed points of the E4M3 format (1 sign, 4 exponent bits biased by 7, 3 mantissa bits,
    no infinities): zero, the smallest subnormal 2^-9, the largest subnormal 7 * 2^-9, the smallest
    normal 2^-6, one, the largest finite value 448, and the two NaN codes."""
    codes = [0x00, 0x01, 0x07, 0x08, 0x38, 0x7E, 0xFE, 0xB8, 0x7F, 0xFF]
    got = oracle_mod.e4m3_to_f64(np.array(codes, dtype=np.uint8))
    want = [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 448.0, -448.0, -1.0]
    assert list(got[:8]) == want
    assert np.isnan(got[8]) and np.isnan(got[9])


def test_fp8_decode_at_unit_scales_equals_the_bf16_decode(oracle_mod):
    """Every finite E4M3 value is exact in bf16, so at unit scales the FP8 decode is the bf16 decode
    of the widened cache, bit for bit."""
    x = inputs.make_decode_fp8(3, 8, 2, 16, 11, seqlens=[11, 4, 0], seed=51, k_scale=1.0, v_scale=1.0)
    got = oracle_mod.decode_fp8(x.q, x.k_cache, x.v_cache, 1.0, 1.0, x.seqlens, x.scale)
    kb = x.k_cache.view(torch.float8_e4m3fn).to(torch.bfloat16)
    vb = x.v_cache.view(torch.float8_e4m3fn).to(torch.bfloat16)
    ref = oracle_mod.decode(x.q, kb, vb, x.seqlens, x.scale)
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (6, 1)])
def test_fp8_decode_with_scales_equals_library_sdpa(oracle_mod, Hq, Hkv):
    """Keys scale the scores and values scale the output: torch SDPA in fp64 on the dequantised
    cache (torch's E4M3 conversion times the per-tensor scales)."""
    d, T = 16, 10
    lens = [10, 3]
    ks, vs = 0.0213, 0.37
    x = inputs.make_decode_fp8(2, Hq, Hkv, d, T, seqlens=lens, seed=52 + Hq, k_scale=ks, v_scale=vs)
    got = oracle_mod.decode_fp8(x.q, x.k_cache, x.v_cache, ks, vs, x.seqlens, x.scale)
    g = Hq // Hkv
    k = torch.from_numpy(_e4m3_f64(x.k_cache.numpy())) * ks
    v = torch.from_numpy(_e4m3_f64(x.v_cache.numpy())) * vs
    for b, n in enumerate(lens):
        q = x.q[b].double()[:, None, :]
        kk = k[b, :n].transpose(0, 1).repeat_interleave(g, dim=0)
        vv = v[b, :n].transpose(0, 1).repeat_interleave(g, dim=0)
        ref = _sdpa(q, kk, vv, x.scale)[:, 0, :].numpy()
        np.testing.assert_allclose(got[b], ref, rtol=1e-12, atol=1e-13)


def test_fp8_rows_past_the_history_are_never_read(oracle_mod):
    x = inputs.make_decode_fp8(2, 8, 2, 16, 12, seqlens=[5, 12], seed=53, poison=True)
    y = inputs.make_decode_fp8(2, 8, 2, 16, 12, seqlens=[5, 12], seed=53, poison=False)
    a = oracle_mod.decode_fp8(x.q, x.k_cache, x.v_cache, x.k_scale, x.v_scale, x.seqlens, x.scale)
    b = oracle_mod.decode_fp8(y.q, y.k_cache, y.v_cache, y.k_scale, y.v_scale, y.seqlens, y.scale)
    assert np.isfinite(a).all()
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------- causal prefill backward


def test_backward_equals_autograd_of_the_repeated_form(oracle_mod):
    """The pages' reference for the backward: repeat K and V along the query-head axis, run plain
    attention, and let differentiation sum the repeats back (torch autograd in fp64), at the pages'
    12/3 equivalence shape with distinct heads."""
    B, S, Hq, Hkv, d = 2, 9, 12, 3, 16
    x = inputs.make_prefill(B, S, Hq, Hkv, d, seed=61)
    dout = inputs.make_dout(B, S, Hq, d, seed=61)
    dq, dk, dv = oracle_mod.prefill_backward(x.q, x.k, x.v, dout, x.scale)
    q = x.q.double().requires_grad_()
    k = x.k.double().requires_grad_()
    v = x.v.double().requires_grad_()
    g = Hq // Hkv
    out = _sdpa(q.transpose(1, 2), k.repeat_interleave(g, dim=2).transpose(1, 2),
                v.repeat_interleave(g, dim=2).transpose(1, 2), x.scale, causal=True).transpose(1, 2)
    out.backward(dout.double())
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=1e-10, atol=1e-12)


def _causal_gqa_forward_np(q, k, v, scale):
    """Plain float64 restatement of the causal grouped forward for finite differences."""
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            for r in range(S):
                s = np.array([scale * q[b, r, h] @ k[b, t, kv] for t in range(r + 1)])
                w = np.exp(s - s.max())
                out[b, r, h] = (w[:, None] * v[b, :r + 1, kv]).sum(0) / w.sum()
    return out


def test_backward_finite_differences(oracle_mod):
    """Central differences of L = sum(dO * out) with respect to every input element."""
    B, S, Hq, Hkv, d = 1, 5, 4, 2, 3
    x = inputs.make_prefill(B, S, Hq, Hkv, d, seed=62)
    dout = inputs.make_dout(B, S, Hq, d, seed=62)
    dq, dk, dv = oracle_mod.prefill_backward(x.q, x.k, x.v, dout, x.scale)
    q0, k0, v0, w = (t.double().numpy() for t in (x.q, x.k, x.v, dout))
    h = 1e-6

    def loss(qq, kk, vv):
        return float((w * _causal_gqa_forward_np(qq, kk, vv, x.scale)).sum())

    for name, arr, grad in (("q", q0, dq), ("k", k0, dk), ("v", v0, dv)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += h
            a2[idx] -= h
            args1 = {"q": q0, "k": k0, "v": v0}
            args2 = dict(args1)
            args1[name], args2[name] = a1, a2
            num[idx] = (loss(args1["q"], args1["k"], args1["v"]) - loss(args2["q"], args2["k"], args2["v"])) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_shared_head_gradient_is_the_group_sum(oracle_mod):
    """dK, dV of a shared head = the sum, over its group, of the per-head gradients of the same
    computation written as MHA on explicitly repeated K and V."""
    B, S, Hq, Hkv, d = 2, 7, 8, 2, 16
    x = inputs.make_prefill(B, S, Hq, Hkv, d, seed=63)
    dout = inputs.make_dout(B, S, Hq, d, seed=63)
    g = Hq // Hkv
    dq, dk, dv = oracle_mod.prefill_backward(x.q, x.k, x.v, dout, x.scale)
    kr = x.k.repeat_interleave(g, dim=2).contiguous()
    vr = x.v.repeat_interleave(g, dim=2).contiguous()
    dq1, dk1, dv1 = oracle_mod.prefill_backward(x.q, kr, vr, dout, x.scale)
    np.testing.assert_allclose(dq, dq1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dk, dk1.reshape(B, S, Hkv, g, d).sum(3), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv, dv1.reshape(B, S, Hkv, g, d).sum(3), rtol=1e-12, atol=1e-14)
    # a group of distinct heads does not give g times one head's gradient
    assert not np.allclose(dk, g * dk1.reshape(B, S, Hkv, g, d)[:, :, :, 0])


def test_backward_selected_rows_and_keys_match_the_full_gradient(oracle_mod):
    B, S, Hq, Hkv, d = 1, 11, 6, 2, 8
    x = inputs.make_prefill(B, S, Hq, Hkv, d, seed=64)
    dout = inputs.make_dout(B, S, Hq, d, seed=64)
    full = oracle_mod.prefill_backward(x.q, x.k, x.v, dout, x.scale)
    rows, keys = [0, 5, 10], [0, 3, 10]
    part = oracle_mod.prefill_backward(x.q, x.k, x.v, dout, x.scale, row_sel=rows, key_sel=keys)
    np.testing.assert_array_equal(part[0][:, rows], full[0][:, rows])
    np.testing.assert_array_equal(part[1][:, keys], full[1][:, keys])
    np.testing.assert_array_equal(part[2][:, keys], full[2][:, keys])
    assert not part[0][:, 1].any() and not part[1][:, 1].any()
    # late keys only: the row statistics are then taken for the selected rows and the rows after the keys
    rows, keys = [1, 4], [7, 10]
    part = oracle_mod.prefill_backward(x.q, x.k, x.v, dout, x.scale, row_sel=rows, key_sel=keys)
    np.testing.assert_array_equal(part[0][:, rows], full[0][:, rows])
    np.testing.assert_array_equal(part[1][:, keys], full[1][:, keys])
    np.testing.assert_array_equal(part[2][:, keys], full[2][:, keys])


# ---------------------------------------------------------------- MLA decode (absorbed weights)


def test_mla_absorbed_decode_equals_explicit_heads(oracle_mod):
    """The weight-absorption identity of the MLA page, with its decoupled RoPE part: per head, attention
    with the key and value rebuilt from the latent (k = c W_uk, v = c W_uv, the RoPE parts appended to
    query and key) equals the oracle's latent-space decode followed by W_uv.  The up-projection W_uk and
    the per-head queries are small integers, so the absorbed query W_uk q is exact in bf16 and both sides
    see the same numbers."""
    g = torch.Generator().manual_seed(31)
    T, d_c, d_r, n_h, d_h = 7, 16, 4, 4, 8
    bf = lambda x: x.to(torch.bfloat16).double()
    c = bf(torch.randn(T, d_c, generator=g, dtype=torch.float64))            # cached latents
    k_r = bf(torch.randn(T, d_r, generator=g, dtype=torch.float64))          # shared RoPE key
    W_uk = torch.randint(-1, 2, (n_h, d_c, d_h), generator=g).double()
    W_uv = torch.randn(n_h, d_c, d_h, generator=g, dtype=torch.float64) / 4
    q = torch.randint(-3, 4, (n_h, d_h), generator=g).double()               # the step's query per head
    q_r = bf(torch.randn(n_h, d_r, generator=g, dtype=torch.float64))
    scale = 1.0 / math.sqrt(d_h + d_r)
    # explicit: each head's own key and value rows
    naive = torch.empty(n_h, d_h, dtype=torch.float64)
    for i in range(n_h):
        k_i = torch.cat([c @ W_uk[i], k_r], dim=1)
        v_i = c @ W_uv[i]
        p = torch.softmax(k_i @ torch.cat([q[i], q_r[i]]) * scale, dim=0)
        naive[i] = p @ v_i
    # absorbed: the latent-space query per head, attention over the cached rows, then W_uv
    q_lat = torch.einsum("hcd,hd->hc", W_uk, q)
    assert torch.equal(bf(q_lat), q_lat)
    qq = torch.cat([q_lat, q_r], dim=1)[None].to(torch.bfloat16)
    kv = torch.cat([c, k_r], dim=1)[None].to(torch.bfloat16)
    lat = torch.from_numpy(oracle_mod.mla_decode(qq, kv, [T], d_c, scale))[0]
    absorbed = torch.einsum("hc,hcd->hd", lat, W_uv)
    assert torch.allclose(absorbed, naive, rtol=0, atol=1e-12)


def test_mla_decode_equals_library_sdpa(oracle_mod):
    """Every head against the shared rows: key = the whole row, value = its latent part (torch SDPA, fp64)."""
    x = inputs.make_mla_decode(3, 16, 40, d_c=32, d_r=8, seqlens=[40, 17, 1], seed=32, q_gain=2.0)
    out = oracle_mod.mla_decode(x.q, x.kv_cache, x.seqlens, x.d_c, x.scale)
    for b, T in enumerate(x.seqlens.tolist()):
        Q = x.q[b].double()[None, :, None, :]
        K = x.kv_cache[b, :T].double()[None, None].expand(1, 16, T, 40)
        V = x.kv_cache[b, :T, :32].double()[None, None].expand(1, 16, T, 32)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=x.scale)[0, :, 0]
        assert np.allclose(out[b], ref.numpy(), rtol=0, atol=1e-12)


def test_mla_decode_is_mqa_with_the_latent_as_value(oracle_mod):
    """The same numbers through the (separately pinned) decode oracle: one KV head whose key is the whole
    row and whose value is the row with its RoPE part zeroed; the latent part of that output is the MLA
    output and the rest is zero."""
    x = inputs.make_mla_decode(2, 8, 30, d_c=24, d_r=8, seqlens=[30, 11], seed=33)
    out = oracle_mod.mla_decode(x.q, x.kv_cache, x.seqlens, x.d_c, x.scale)
    k = x.kv_cache[:, :, None, :]
    v = k.clone()
    v[..., 24:] = 0
    mqa = oracle_mod.decode(x.q, k, v, x.seqlens, x.scale)
    assert np.allclose(mqa[..., :24], out, rtol=0, atol=1e-13)
    assert np.all(mqa[..., 24:] == 0)


def test_mla_decode_closed_forms(oracle_mod):
    """One cached token returns its latent part; an empty history gives zeros; a zero query averages the
    latents; the RoPE part of the key moves the weights (two rows alike in the latent, apart in RoPE)."""
    x = inputs.make_mla_decode(3, 4, 5, d_c=8, d_r=4, seqlens=[1, 0, 5], seed=34)
    out = oracle_mod.mla_decode(x.q, x.kv_cache, x.seqlens, x.d_c, x.scale)
    assert np.array_equal(out[0], np.broadcast_to(x.kv_cache[0, 0, :8].double().numpy(), (4, 8)))
    assert np.all(out[1] == 0)
    q0 = torch.zeros_like(x.q)
    z = oracle_mod.mla_decode(q0, x.kv_cache, x.seqlens, x.d_c, x.scale)
    assert np.allclose(z[2], x.kv_cache[2, :5, :8].double().mean(0).numpy(), rtol=0, atol=1e-14)
    kv = torch.zeros(1, 2, 12, dtype=torch.bfloat16)
    kv[0, 0, :8] = 1.0
    kv[0, 1, :8] = -1.0
    kv[0, 1, 8] = 4.0                      # only the second row's RoPE key matches the query
    qq = torch.zeros(1, 1, 12, dtype=torch.bfloat16)
    qq[0, 0, 8] = 1.0
    o = oracle_mod.mla_decode(qq, kv, [2], 8, 1.0)
    w1 = math.exp(4.0) / (1.0 + math.exp(4.0))
    assert np.allclose(o[0, 0], (1 - w1) * 1.0 + w1 * -1.0, rtol=0, atol=1e-14)


def test_mla_cache_bytes_per_token(oracle_mod):
    """The MLA page's cache sizes (tests/golden/mla.txt): 512 + 64 numbers per token and layer against
    2 x 128 heads x 128 for MHA (about 1/57), and DeepSeek-V3's 61 layers of 576 bf16 numbers per token.
    The latent is both key and value, so the cache holds one row where the GQA byte model counts a
    separate K and V: half of kv_bytes for one KV head of width 576."""
    g = {ln.split()[0]: int(ln.split()[1]) for ln in _lines("mla.txt")}
    mha, mla = 2 * 128 * 128, 512 + 64
    assert g["mha_numbers_per_token_layer"] == mha and g["mla_numbers_per_token_layer"] == mla
    assert round(mha / mla) == g["mla_fraction_of_mha"]
    assert 2 * g["deepseek_v3_bytes_per_token"] == oracle_mod.kv_bytes(61, 1, 1, 576, 2)

