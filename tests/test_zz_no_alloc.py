"""gqa_decode_noalloc through the C ABI: same results as gqa_decode, no device allocation.

The entry point exists for callers that cannot let a library allocate device
memory (a serving engine whose pool already holds the GPU, a decode loop that
cannot absorb cudaMalloc).  Its split partials live in a fixed 32 MiB array
inside libgqa.so.  This file is collected last so that a run stopping at the
first failure has already run every other test; it also passes on its own in
a fresh process.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import grouped_query_attention_02_b200 as gqa
from grouped_query_attention_02_b200 import inputs
from tests._tolerance import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _call_noalloc(lib, x, out):
    B, Hq, d = x.q.shape
    _, Tmax, Hkv, _ = x.k_cache.shape
    return lib.gqa_decode_noalloc(x.q.data_ptr(), x.k_cache.data_ptr(), x.v_cache.data_ptr(), x.seqlens.data_ptr(),
                                  B, Hq, Hkv, d, Tmax, ctypes.c_float(x.scale), out.data_ptr(),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


SHAPES = [
    # (B, Hq, Hkv, Tmax, seqlens): the second splits the history, so the scratch really holds partials
    (1, 8, 2, 256, None),
    (8, 32, 8, 8192, [8192, 8000, 4097, 64, 1, 0, 3000, 8191]),
    (3, 32, 2, 20000, [20000, 12345, 777]),
    # the CUDA-core kernel's group sizes: MHA and groups of two, each split over several pieces
    (2, 16, 16, 12000, [12000, 5000]),
    (2, 16, 8, 12000, [11999, 130]),
]
IDS = ["tiny", "split-8x8192", "group16-split", "mha-split", "group2-split"]


@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_matches_gqa_decode_and_the_oracle_on_two_calls_in_a_row(oracle_mod, shape):
    B, Hq, Hkv, Tmax, lens = shape
    lib = gqa.load()
    x = inputs.make_decode(B, Hq, Hkv, 128, Tmax, seqlens=lens, device=DEV, seed=77)
    ref = gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    torch.cuda.synchronize()
    ref64 = ref.double().cpu().numpy()
    exact = oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens.cpu(), x.scale)
    for call in range(2):
        out = torch.full_like(x.q, float("nan"))
        assert _call_noalloc(lib, x, out) == 0
        torch.cuda.synchronize()
        assert gqa.gqa_get_last_device_status() == 0
        got = out.double().cpu().numpy()
        assert_close(got, ref64)      # the existing entry point, at the decode gates
        assert_close(got, exact)      # and the fp64 oracle directly
    if B == 8:
        assert gqa.gqa_decode_plan(B, Hq, Hkv, 128, Tmax, torch.cuda.get_device_properties(0).multi_processor_count)[1] > 1


def test_allocates_nothing(oracle_mod):
    """With the library's workspace handed back and an allocator installed that refuses every request,
    the call still succeeds (it never asks), device memory does not change, and the result is right."""
    lib = gqa.load()
    x = inputs.make_decode(4, 32, 4, 128, 9000, seqlens=[9000, 8191, 33, 4500], device=DEV, seed=78)
    out = torch.full_like(x.q, float("nan"))
    torch.cuda.synchronize()
    gqa.gqa_release()
    asked = []
    gqa.gqa_set_workspace_allocator(lambda n, dev: asked.append(n) or 0, lambda p, n, dev: None)
    try:
        # the first call of a fresh process also loads the kernels' code (the driver's doing, not an
        # allocation by the library), so free memory is sampled after it
        assert _call_noalloc(lib, x, out) == 0
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        for _ in range(2):
            assert _call_noalloc(lib, x, out) == 0
            torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert asked == []
        assert free1 == free0
        assert gqa.gqa_get_last_device_status() == 0
        # the library's own entry point does ask, and is refused
        with pytest.raises(gqa.GQAError):
            gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
        assert asked
    finally:
        gqa.gqa_set_workspace_allocator(None, None)
    assert_close(out.double().cpu().numpy(), oracle_mod.decode(x.q, x.k_cache, x.v_cache, x.seqlens.cpu(), x.scale))


def test_rejects_partials_larger_than_the_fixed_scratch(oracle_mod):
    # 2048 sequences x 32 query heads: even one piece per sequence needs 2048*32*130*4 B = 34 MB of
    # partials, more than the 32 MiB array (a cache of 1024 tokens is planned on the device; caches of
    # at most 512 run as one launch with no partials at all, and are accepted)
    B, Hq, Hkv, Tmax = 2048, 32, 8, 1024
    assert B * Hq * (128 + 2) * 4 > 32 << 20
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device=DEV)
    k = torch.empty((B, Tmax, Hkv, 128), dtype=torch.bfloat16, device=DEV)
    v = torch.empty_like(k)
    sl = torch.full((B,), Tmax, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    lib = gqa.load()
    st = lib.gqa_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(), B, Hq, Hkv, 128, Tmax,
                                ctypes.c_float(0.088), out.data_ptr(), None)
    assert st == 2, gqa.gqa_status_string(st)
    assert gqa.gqa_last_launch_count() == 0
    # the same batch over a 512-token cache needs no scratch: one launch, right answer
    Tmax = 512
    x = inputs.make_decode(B, Hq, Hkv, 128, Tmax, device=DEV, seed=79)
    assert _call_noalloc(lib, x, out) == 0
    torch.cuda.synchronize()
    assert gqa.gqa_last_launch_count() == 1 and gqa.gqa_get_last_device_status() == 0
    bs = [0, 1000, 2047]
    ref = oracle_mod.decode(x.q[bs].cpu(), x.k_cache[bs].cpu(), x.v_cache[bs].cpu(), x.seqlens[bs].cpu(), x.scale)
    assert_close(out[bs].double().cpu().numpy(), ref)
