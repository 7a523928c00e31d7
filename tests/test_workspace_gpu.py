"""The library workspace from a caller's allocator (gqa_set_workspace_allocator), on the GPU.

A failing allocator is how workspace exhaustion is provoked: the call must return
GQA_ERR_OUT_OF_MEMORY with nothing enqueued and the library must keep working once a
working allocator is back.  A pool-backed allocator must actually be used, and every
block it gave must be handed back when the allocator changes.
"""
from __future__ import annotations

import pytest
import torch

import grouped_query_attention_02_b200 as gqa
from grouped_query_attention_02_b200 import inputs
from tests._tolerance import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
OOM, MISALIGNED = 4, 3


def _split_history():
    # two long histories: the decode plans several pieces per history and needs split partials
    return inputs.make_decode(2, 8, 2, 128, 20000, seqlens=[20000, 9001], device=DEV, seed=4)


def _ref(oracle_mod, x):
    return oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens.cpu(), x.scale)


def test_failing_allocator_reports_out_of_memory_and_enqueues_nothing(oracle_mod):
    x = _split_history()
    gqa.gqa_release()
    asked = []
    gqa.gqa_set_workspace_allocator(lambda n, dev: asked.append(n) or 0, lambda p, n, dev: None)
    try:
        out = torch.full_like(x.q, 7.0)
        torch.cuda.synchronize()
        with pytest.raises(gqa.GQAError) as e:
            gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, out=out)
        assert e.value.status == OOM and asked and asked[0] > 0
        assert gqa.gqa_last_launch_count() == 0
        # the backward's row statistics come from the workspace as well
        p = inputs.make_prefill(1, 256, 8, 2, 128, device=DEV, seed=2)
        o, lse = gqa.gqa_prefill_causal_fwd(p.q, p.k, p.v)
        dout = inputs.make_dout(1, 256, 8, 128, device=DEV, seed=2)
        with pytest.raises(gqa.GQAError) as e:
            gqa.gqa_prefill_causal_bwd(p.q, p.k, p.v, o, lse, dout)
        assert e.value.status == OOM
        torch.cuda.synchronize()
        assert torch.all(out == 7.0)
    finally:
        gqa.gqa_set_workspace_allocator(None, None)
    out = gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    torch.cuda.synchronize()
    assert_close(out.double().cpu().numpy(), _ref(oracle_mod, x))


def test_workspace_comes_from_the_callers_pool(oracle_mod):
    x = _split_history()
    gqa.gqa_release()
    blocks, log = {}, []

    def alloc(n, dev):
        t = torch.empty(n + 256, dtype=torch.uint8, device=f"cuda:{dev}")
        p = (t.data_ptr() + 255) // 256 * 256
        blocks[p] = t
        log.append(("alloc", n))
        return p

    def free(p, n, dev):
        log.append(("free", n))
        del blocks[p]

    gqa.gqa_set_workspace_allocator(alloc, free)
    try:
        out = gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
        torch.cuda.synchronize()
        assert_close(out.double().cpu().numpy(), _ref(oracle_mod, x))
        assert len(blocks) == 1 and log[0][0] == "alloc"
        # a larger need grows the workspace: the old block goes back before the new one is used
        p = inputs.make_prefill(1, 8192, 32, 8, 128, device=DEV, seed=3)
        o, lse = gqa.gqa_prefill_causal_fwd(p.q, p.k, p.v)
        dout = inputs.make_dout(1, 8192, 32, 128, device=DEV, seed=3)
        gqa.gqa_prefill_causal_bwd(p.q, p.k, p.v, o, lse, dout)
        torch.cuda.synchronize()
        if log[-1][1] > log[0][1]:
            assert [k for k, _ in log[-2:]] == ["free", "alloc"] and len(blocks) == 1
    finally:
        gqa.gqa_set_workspace_allocator(None, None)
    assert not blocks and log[-1][0] == "free"
    out2 = gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_misaligned_block_is_handed_back():
    x = _split_history()
    gqa.gqa_release()
    blocks = {}

    def alloc(n, dev):
        t = torch.empty(n + 512, dtype=torch.uint8, device=f"cuda:{dev}")
        p = (t.data_ptr() + 255) // 256 * 256 + 16
        blocks[p] = t
        return p

    gqa.gqa_set_workspace_allocator(alloc, lambda p, n, dev: blocks.pop(p))
    try:
        with pytest.raises(gqa.GQAError) as e:
            gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
        assert e.value.status == MISALIGNED and not blocks
    finally:
        gqa.gqa_set_workspace_allocator(None, None)
