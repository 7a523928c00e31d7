"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and its host-side logic (argument checks, split plan, byte counts) behaves.

Argument checks run before any CUDA call, so the pointers handed over here
are never dereferenced.
"""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import grouped_query_attention_02_b200 as gqa
from grouped_query_attention_02_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, OOM, CUDA, TIMEOUT = range(7)


@pytest.fixture(scope="module")
def lib():
    from grouped_query_attention_02_b200 import build

    build.build()
    return gqa.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in gqa.h but not exported by libgqa.so"
    assert set(names) == set(gqa.EXPORTS), "binding and header disagree"


def test_binding_mirrors_header_names():
    for n in _declared():
        assert hasattr(gqa, n), f"binding lacks {n}"


def test_status_strings(lib):
    for s in range(7):
        assert gqa.gqa_status_string(s)
    assert gqa.gqa_status_string(TIMEOUT) != gqa.gqa_status_string(OK)
    assert gqa.gqa_version().startswith("gqa-b200")


A = 0x10000          # a 16-byte aligned fake address (never dereferenced)
U = 0x10008          # not 16-byte aligned


def _decode(lib, q=A, k=A, v=A, sl=A, B=2, Hq=8, Hkv=2, d=128, T=64, out=A):
    return lib.gqa_decode(q, k, v, sl, B, Hq, Hkv, d, T, ctypes.c_float(0.088), out, None)


def test_decode_argument_checks(lib):
    assert _decode(lib, q=None) == INVALID
    assert _decode(lib, sl=None) == INVALID
    assert _decode(lib, out=None) == INVALID
    assert _decode(lib, B=0) == INVALID
    assert _decode(lib, Hq=0) == INVALID
    assert _decode(lib, T=0) == INVALID
    assert _decode(lib, Hq=6, Hkv=4) == INVALID          # irregular grouping
    assert _decode(lib, d=64) == UNSUPPORTED
    assert _decode(lib, q=U) == MISALIGNED
    assert _decode(lib, k=U) == MISALIGNED
    assert _decode(lib, out=U) == MISALIGNED
    assert _decode(lib, sl=A + 2) == MISALIGNED
    assert gqa.gqa_last_launch_count() == 0


def test_expanded_and_prefill_argument_checks(lib):
    f = ctypes.c_float(0.088)
    assert lib.gqa_decode_expanded(A, A, A, A, 2, 8, 2, 128, 64, f, A, None, A, None) == INVALID
    assert lib.gqa_decode_expanded(A, A, A, A, 2, 8, 2, 128, 64, f, A, U, A, None) == MISALIGNED
    assert lib.gqa_prefill_causal(A, A, A, 2, 64, 8, 3, 128, A, None) == INVALID
    assert lib.gqa_prefill_causal(A, A, A, 2, 0, 8, 2, 128, A, None) == INVALID
    assert lib.gqa_prefill_causal(A, A, A, 2, 64, 8, 2, 96, A, None) == UNSUPPORTED
    assert lib.gqa_prefill_causal(A, A, U, 2, 64, 8, 2, 128, A, None) == MISALIGNED
    assert lib.gqa_selftest_wait_timeout(0, None) == INVALID
    assert lib.gqa_set_profile_events(A, None) == INVALID


def test_expanded_bytes(lib):
    assert gqa.gqa_decode_expanded_bytes(49, 8192, 32, 128) == 49 * 8192 * 32 * 128 * 2
    assert gqa.gqa_decode_expanded_bytes(0, 8192, 32, 128) == 0


@pytest.mark.parametrize("w", workloads.DECODE_WORKLOADS, ids=lambda w: w.name)
def test_split_plan_covers_the_history(lib, w):
    chunk, nsplit, ws = gqa.gqa_decode_plan(w.B, w.Hq, w.Hkv, w.d, w.Tmax, 148)
    assert chunk % 64 == 0 and chunk > 0
    assert nsplit * chunk >= w.Tmax and (nsplit - 1) * chunk < w.Tmax
    partials = w.B * w.Hq * nsplit * (128 + 2) * 4
    if 3 <= w.group <= 32 and (w.Tmax + 127) // 128 <= 4:
        # a cache of at most four tiles: one launch over whole histories, no workspace
        assert nsplit == 1 and ws == 0
    elif 3 <= w.group <= 32:
        # tensor-core path: pieces are cut on the device from the real lengths (at most nsplit per
        # sequence); the workspace also holds the piece list
        assert ws >= partials
    else:
        assert ws == (partials if nsplit > 1 else 0)


def test_split_plan_fills_the_machine(lib):
    # 392 (sequence, kv head) tiles on 296 CTA slots: one split alone would leave a 1.3-wave tail
    chunk, nsplit, _ = gqa.gqa_decode_plan(49, 32, 8, 128, 8192, 148)
    assert nsplit > 1
    # 32 tiles of 131072 tokens: the history must be split many ways
    chunk, nsplit, _ = gqa.gqa_decode_plan(16, 32, 2, 128, 131072, 148)
    assert nsplit >= 8
    # a tiny history stays in one split
    assert gqa.gqa_decode_plan(1, 8, 2, 128, 64, 148)[1] == 1


def test_plan_argument_checks(lib):
    c, n, w = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    assert lib.gqa_decode_plan(1, 8, 3, 128, 64, 148, ctypes.byref(c), ctypes.byref(n), ctypes.byref(w)) == INVALID
    assert lib.gqa_decode_plan(1, 8, 2, 128, 64, 0, ctypes.byref(c), ctypes.byref(n), ctypes.byref(w)) == INVALID
    assert lib.gqa_decode_plan(1, 8, 2, 64, 64, 148, ctypes.byref(c), ctypes.byref(n), ctypes.byref(w)) == UNSUPPORTED


def _decode_fp8(lib, q=A, k=A, v=A, sl=A, B=2, Hq=8, Hkv=2, d=128, T=64, out=A, scale=0.088, ks=0.01, vs=0.02):
    return lib.gqa_decode_fp8(q, k, v, sl, B, Hq, Hkv, d, T, ctypes.c_float(scale), ctypes.c_float(ks),
                              ctypes.c_float(vs), out, None)


def test_fp8_decode_argument_checks(lib):
    assert _decode_fp8(lib, k=None) == INVALID
    assert _decode_fp8(lib, B=0) == INVALID
    assert _decode_fp8(lib, Hq=6, Hkv=4) == INVALID
    assert _decode_fp8(lib, ks=float("nan")) == INVALID
    assert _decode_fp8(lib, vs=float("inf")) == INVALID
    assert _decode_fp8(lib, scale=float("inf")) == INVALID
    assert _decode_fp8(lib, d=64) == UNSUPPORTED
    assert _decode_fp8(lib, Hq=64, Hkv=1) == UNSUPPORTED     # groups above 32
    assert _decode_fp8(lib, v=U) == MISALIGNED
    assert gqa.gqa_last_launch_count() == 0


def test_prefill_fwd_and_bwd_argument_checks(lib):
    assert lib.gqa_prefill_causal_fwd(A, A, A, 2, 64, 8, 2, 128, A, None, None) == INVALID
    assert lib.gqa_prefill_causal_fwd(A, A, A, 2, 64, 8, 2, 128, A, A + 2, None) == MISALIGNED
    assert lib.gqa_prefill_causal_fwd(A, A, A, 2, 64, 8, 3, 128, A, A, None) == INVALID
    bwd = lambda **kw: lib.gqa_prefill_causal_bwd(
        kw.get("q", A), A, A, A, kw.get("lse", A), kw.get("dout", A), 2, 64, 8, kw.get("Hkv", 2), kw.get("d", 128),
        kw.get("dq", A), A, A, None)
    assert bwd(dout=None) == INVALID
    assert bwd(lse=None) == INVALID
    assert bwd(Hkv=3) == INVALID
    assert bwd(d=96) == UNSUPPORTED
    assert bwd(dq=U) == MISALIGNED
    assert gqa.gqa_last_launch_count() == 0


def test_workspace_allocator_comes_in_pairs(lib):
    keep = (gqa.ALLOC_FN(lambda n, dev, ctx: None), gqa.FREE_FN(lambda p, n, dev, ctx: None))
    fn, fr = (ctypes.cast(f, ctypes.c_void_p) for f in keep)
    assert lib.gqa_set_workspace_allocator(fn, None, None) == INVALID
    assert lib.gqa_set_workspace_allocator(None, fr, None) == INVALID
    assert lib.gqa_set_workspace_allocator(None, None, None) == OK
    with pytest.raises(ValueError):
        gqa.gqa_set_workspace_allocator(lambda n, dev: 0, None)


def test_mla_decode_argument_checks(lib):
    f = lambda q=A, kv=A, sl=A, B=2, Hq=16, dc=512, dr=64, T=64, out=A: lib.gqa_mla_decode(
        q, kv, sl, B, Hq, dc, dr, T, ctypes.c_float(0.07), out, None)
    assert f(q=None) == INVALID and f(kv=None) == INVALID and f(sl=None) == INVALID and f(out=None) == INVALID
    assert f(B=0) == INVALID and f(Hq=0) == INVALID and f(T=0) == INVALID and f(dr=-1) == INVALID
    assert f(dc=128) == UNSUPPORTED and f(dr=0) == UNSUPPORTED and f(B=70000) == UNSUPPORTED
    assert f(q=U) == MISALIGNED and f(kv=U) == MISALIGNED and f(out=U) == MISALIGNED

