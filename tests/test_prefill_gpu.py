"""GPU parity of the tcgen05 causal prefill against the fp64 oracle, through the C ABI."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import grouped_query_attention_02_b200 as gqa
from grouped_query_attention_02_b200 import inputs, workloads
from tests._tolerance import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(p):
    out = gqa.gqa_prefill_causal(p.q, p.k, p.v)
    torch.cuda.synchronize()
    assert gqa.gqa_get_last_device_status() == 0
    return out


def _check_all(oracle_mod, p, out, abs_bar=True):
    ref = oracle_mod.prefill_causal(p.q, p.k, p.v, p.scale)
    return assert_close(out.double().cpu().numpy(), ref, kind="prefill", vmax=float(p.v.abs().max()),
                        abs_bar=abs_bar)


def test_small_prefill_full(oracle_mod):
    p = inputs.make_prefill(1, 256, 8, 2, 128, device=DEV, seed=0)
    _check_all(oracle_mod, p, _run(p))


def test_pages_equivalence_shape(oracle_mod):
    # two sequences of 9 tokens, 12 query heads over 3 KV heads (the pages' check), at d = 128
    p = inputs.make_prefill(2, 9, 12, 3, 128, device=DEV, seed=1)
    _check_all(oracle_mod, p, _run(p))


@pytest.mark.parametrize("S", [1, 2, 127, 128, 129, 300, 513])
def test_ragged_lengths(oracle_mod, S):
    p = inputs.make_prefill(2, S, 8, 2, 128, device=DEV, seed=10 + S)
    _check_all(oracle_mod, p, _run(p))


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 1), (6, 2), (32, 8), (32, 2), (71, 1)])
def test_group_sizes(oracle_mod, Hq, Hkv):
    p = inputs.make_prefill(1, 384, Hq, Hkv, 128, device=DEV, seed=Hq * 7 + Hkv)
    _check_all(oracle_mod, p, _run(p))


def test_peaky_scores_move_the_running_maximum(oracle_mod):
    # q scaled by 8: nearly one-hot weights, outputs up to |v| ~ 5 where the bf16 output step is 2^-5
    p = inputs.make_prefill(2, 640, 8, 2, 128, device=DEV, seed=3, q_gain=8.0)
    _check_all(oracle_mod, p, _run(p), abs_bar=False)


def test_grouped_equals_expanded_heads(oracle_mod):
    # physically repeating K/V (MHA over the copies) must give the same answer as the grouped call
    p = inputs.make_prefill(2, 300, 12, 3, 128, device=DEV, seed=4)
    out_g = _run(p)
    p_rep = inputs.PrefillInputs(p.q, p.k.repeat_interleave(4, dim=2).contiguous(),
                                 p.v.repeat_interleave(4, dim=2).contiguous(), p.scale)
    out_e = _run(p_rep)
    assert torch.equal(out_g, out_e)


def test_causal_prefill_workload_sampled(oracle_mod):
    w = workloads.CAUSAL_PREFILL
    p = inputs.make_prefill(w.B, w.S, w.Hq, w.Hkv, w.d, device=DEV, seed=0)
    out = _run(p)
    g = torch.Generator().manual_seed(5)
    rows = []
    edges = [0, 1, 2, 127, 128, 129, 255, 256, 4095, 4096, 4097, 8063, 8064, 8190, 8191]
    for b in range(w.B):
        for h in (0, 3, 4, 17, 31):
            rr = edges + torch.randint(0, w.S, (6,), generator=g).tolist()
            rows += [(b, h, r) for r in rr]
    ref = oracle_mod.prefill_causal(p.q, p.k, p.v, p.scale, rows=rows)
    got = np.stack([out[b, r, h].double().cpu().numpy() for b, h, r in rows])
    assert_close(got, ref, kind="prefill", vmax=float(p.v.abs().max()))


def test_deterministic_and_stream_ordered():
    p = inputs.make_prefill(2, 1024, 32, 8, 128, device=DEV, seed=6)
    a = _run(p).clone()
    s = torch.cuda.Stream()
    out = torch.full_like(p.q, float("nan"))
    with torch.cuda.stream(s):
        gqa.gqa_prefill_causal(p.q, p.k, p.v, out=out, stream=s)
    s.synchronize()
    assert torch.equal(a, out)
