"""Host logic of the split planner (no GPU): the workspace budget bounds the split partials on both
kernel families.  A call of gqa_decode_noalloc plans with its fixed 32 MiB array as the budget; shapes
whose partials fit with fewer pieces per sequence must get such a plan, not a refusal.  The shapes
below need caches of over 100 GB, which is why this is checked on the planner itself."""
from __future__ import annotations

import ctypes

import pytest

import grouped_query_attention_02_b200 as gqa

MANGLED = "_ZN3gqa16decode_plan_hostEiiiiimb"   # gqa::decode_plan_host(int, int, int, int, int, size_t, bool)
NOALLOC_BUDGET = (32 << 20) - (1 << 20)         # the array less the room the plan's bookkeeping takes


class Plan(ctypes.Structure):
    _fields_ = [("tile", ctypes.c_int), ("chunk", ctypes.c_int), ("nsplit", ctypes.c_int), ("hb", ctypes.c_int),
                ("nhb", ctypes.c_int), ("tensor_cores", ctypes.c_bool), ("off_hdr", ctypes.c_size_t),
                ("off_nsb", ctypes.c_size_t), ("off_items", ctypes.c_size_t), ("off_po", ctypes.c_size_t),
                ("off_pml", ctypes.c_size_t), ("ws_bytes", ctypes.c_size_t), ("static_plan", ctypes.c_bool)]


@pytest.fixture(scope="module")
def plan():
    lib = gqa.load()
    f = getattr(lib, MANGLED)
    f.restype = Plan
    f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_size_t, ctypes.c_bool]
    return lambda B, Hq, Hkv, T, budget: f(B, Hq, Hkv, T, 148, budget, False)


@pytest.mark.parametrize("B,Hq,Hkv,T", [(256, 64, 32, 32768), (1024, 32, 16, 32768)])
def test_cuda_core_plan_respects_the_budget(plan, B, Hq, Hkv, T):
    # group sizes 2 (CUDA-core kernel): with the library's 256 MiB budget the plan splits and its
    # partials exceed the no-alloc array; with the array's budget it keeps one piece per sequence
    big = plan(B, Hq, Hkv, T, 256 << 20)
    assert not big.tensor_cores and big.nsplit > 1 and big.ws_bytes > 32 << 20
    small = plan(B, Hq, Hkv, T, NOALLOC_BUDGET)
    assert small.nsplit >= 1 and small.ws_bytes <= NOALLOC_BUDGET
    assert small.chunk * small.nsplit >= T


@pytest.mark.parametrize("B,Hq,Hkv,T", [(64, 32, 32, 131072), (16, 128, 128, 262144), (8, 64, 32, 65536)])
def test_cuda_core_plan_unchanged_when_it_fits(plan, B, Hq, Hkv, T):
    a = plan(B, Hq, Hkv, T, 256 << 20)
    b = plan(B, Hq, Hkv, T, NOALLOC_BUDGET)
    if a.ws_bytes <= NOALLOC_BUDGET:
        assert (a.nsplit, a.chunk, a.ws_bytes) == (b.nsplit, b.chunk, b.ws_bytes)
    assert b.ws_bytes <= NOALLOC_BUDGET


def test_every_split_the_budget_allows_covers_the_history(plan):
    for budget in (0, 1 << 20, 4 << 20, NOALLOC_BUDGET, 256 << 20):
        for (B, Hq, Hkv, T) in [(4, 16, 16, 100000), (2, 32, 16, 50000), (1, 128, 128, 262144)]:
            p = plan(B, Hq, Hkv, T, budget)
            assert p.nsplit >= 1 and p.chunk * p.nsplit >= T and p.chunk * (p.nsplit - 1) < T
            if p.nsplit > 1:
                assert B * Hq * p.nsplit * (128 + 2) * 4 <= budget


@pytest.mark.parametrize("T,static", [(1, True), (512, True), (513, False), (8192, False)])
def test_short_caches_take_one_launch(plan, T, static):
    # the tensor-core path (group 4): caches of at most four 128-token tiles run without the planner
    # (no workspace at all), longer ones are planned on the device
    p = plan(49, 32, 8, T, 256 << 20)
    assert p.tensor_cores and p.static_plan == static
    assert (p.ws_bytes == 0) == static
    assert p.nsplit >= 1 and p.chunk * p.nsplit >= T
