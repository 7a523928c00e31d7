"""GPU parity of the causal prefill backward (dq, and dk / dv summed over each group) against the
fp64 oracle, through the C ABI.  Small shapes are compared over every gradient element; the
workload shape on sampled query rows (dq) and keys (dk, dv) of one sequence."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import grouped_query_attention_02_b200 as gqa
from grouped_query_attention_02_b200 import inputs, workloads
from tests._tolerance import compare

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(x, dout):
    out, lse = gqa.gqa_prefill_causal_fwd(x.q, x.k, x.v)
    dq, dk, dv = gqa.gqa_prefill_causal_bwd(x.q, x.k, x.v, out, lse, dout)
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    return out, lse, dq, dk, dv


def _check(got, ref, name):
    """The stated bar (normwise relative 2e-2; absolute 2e-2, scaled by max|ref| where gradients exceed 1,
    since rounding a gradient of magnitude m to bf16 alone moves it by up to 2^-8 m) and a tight gate
    from the arithmetic: every product term carries at most about 2^-8 relative error (P or dS rounded
    to bf16, D from the bf16 output), the gradient itself is rounded to bf16, and the terms' absolute
    sum stays within a few times max|ref| here, so |g - r| <= 2^-8 |r| + 2^-7 max(max|ref|, 2^-10)."""
    r_max = float(np.abs(ref).max()) if ref.size else 0.0
    s = compare(got.double().cpu().numpy(), ref, kind="backward", floor=2.0 ** -7 * max(r_max, 2.0 ** -10))
    # both absolute figures stay in the record, so drift toward the unscaled bar is visible
    s["abs_bar_scaled"] = 2e-2 * max(1.0, s["ref_max"])
    s["within_unscaled_abs_bar"] = s["max_abs"] <= 2e-2
    assert s["nan"] == 0, (name, s)
    assert s["rel_normwise"] <= 2e-2 or s["max_abs"] <= 2.0 ** -16, (name, s)
    assert s["max_abs"] <= s["abs_bar_scaled"], (name, s)
    if s["ref_max"] <= 1.0:
        assert s["within_unscaled_abs_bar"], (name, s)
    assert s["tight_violations"] == 0, (name, s)
    return s


def _case(oracle_mod, B, S, Hq, Hkv, seed):
    x = inputs.make_prefill(B, S, Hq, Hkv, 128, device=DEV, seed=seed)
    dout = inputs.make_dout(B, S, Hq, 128, device=DEV, seed=seed)
    out, lse, dq, dk, dv = _run(x, dout)
    rq, rk, rv = oracle_mod.prefill_backward(x.q.cpu(), x.k.cpu(), x.v.cpu(), dout.cpu(), x.scale)
    _check(dq, rq, "dq")
    _check(dk, rk, "dk")
    _check(dv, rv, "dv")


def test_backward_small_ragged(oracle_mod):
    _case(oracle_mod, 2, 300, 8, 2, 71)


@pytest.mark.parametrize("S", [1, 127, 128, 129, 257])
def test_backward_tile_edges(oracle_mod, S):
    _case(oracle_mod, 1, S, 8, 2, 72 + S)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 1), (6, 2), (12, 3), (32, 8)])
def test_backward_group_sizes(oracle_mod, Hq, Hkv):
    _case(oracle_mod, 1, 200, Hq, Hkv, 80 + Hq + Hkv)


def test_forward_lse_matches_the_definition():
    x = inputs.make_prefill(2, 260, 8, 2, 128, device=DEV, seed=90)
    out, lse = gqa.gqa_prefill_causal_fwd(x.q, x.k, x.v)
    ref_out = gqa.gqa_prefill_causal(x.q, x.k, x.v)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    q = x.q.double().cpu().transpose(1, 2)                       # [B,Hq,S,d]
    k = x.k.double().cpu().repeat_interleave(4, dim=2).transpose(1, 2)
    s = q @ k.transpose(-1, -2) * x.scale
    mask = torch.ones(260, 260, dtype=torch.bool).tril()
    ref = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(lse.double().cpu().numpy(), ref.numpy(), rtol=0, atol=2e-5)


def test_backward_workload_sampled(oracle_mod):
    """The causal prefill workload shape (B=4, S=8192, 32 query / 8 KV heads): one sequence, sampled
    query rows for dq and keys near the end for dk / dv (their row statistics stay cheap)."""
    w = workloads.CAUSAL_PREFILL
    x = inputs.make_prefill(w.B, w.S, w.Hq, w.Hkv, w.d, device=DEV, seed=0)
    dout = inputs.make_dout(w.B, w.S, w.Hq, w.d, device=DEV, seed=0)
    out, lse, dq, dk, dv = _run(x, dout)
    rows = [0, 1, 127, 128, 4095, 8190, 8191]
    keys = [8064, 8100, 8190, 8191]
    b = 2
    rq, rk, rv = oracle_mod.prefill_backward(x.q[b:b + 1].cpu(), x.k[b:b + 1].cpu(), x.v[b:b + 1].cpu(),
                                             dout[b:b + 1].cpu(), x.scale, row_sel=rows, key_sel=keys)
    _check(dq[b:b + 1, rows], rq[:, rows], "dq")
    _check(dk[b:b + 1, keys], rk[:, keys], "dk")
    _check(dv[b:b + 1, keys], rv[:, keys], "dv")


def test_backward_deterministic():
    x = inputs.make_prefill(1, 700, 8, 2, 128, device=DEV, seed=91)
    dout = inputs.make_dout(1, 700, 8, 128, device=DEV, seed=91)
    a = _run(x, dout)
    b = _run(x, dout)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    assert gqa.gqa_last_launch_count() == 2   # the dQ kernel (which also forms D), then dK/dV


def test_backward_repeated_long_sequence():
    """Many key tiles per CTA (S = 8192: up to 64 per dQ CTA and 64 query tiles per dK/dV CTA), run
    repeatedly: every run ends with the device status clear (no bounded wait gave up, as a handshake whose
    phase a fast warpgroup could complete twice before its waiter looks would make one) and every run
    gives the same bits."""
    x = inputs.make_prefill(1, 8192, 8, 2, 128, device=DEV, seed=97)
    dout = inputs.make_dout(1, 8192, 8, 128, device=DEV, seed=97)
    out, lse = gqa.gqa_prefill_causal_fwd(x.q, x.k, x.v)
    first = None
    for _ in range(12):
        grads = gqa.gqa_prefill_causal_bwd(x.q, x.k, x.v, out, lse, dout)
        torch.cuda.synchronize()
        assert gqa.gqa_get_last_device_status() == 0
        if first is None:
            first = [g.clone() for g in grads]
        else:
            for u, v in zip(first, grads):
                assert torch.equal(u, v)
