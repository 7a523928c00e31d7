"""B200-native grouped-query attention: decode and causal prefill behind a C ABI.

This module is the thin Python binding of ``libgqa.so`` (``include/gqa.h``):
it checks tensor dtypes/shapes/devices, passes raw pointers, sizes and the
current CUDA stream through ctypes, and turns status codes into exceptions.
Every step of the computation runs in the library's CUDA kernels; there is no
fallback.  If the library is missing the first call raises ``RuntimeError``.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "GQAError", "gqa_decode", "gqa_decode_fp8", "gqa_decode_noalloc", "gqa_prefill_causal",
    "gqa_prefill_causal_fwd", "gqa_prefill_causal_bwd", "gqa_decode_expanded", "gqa_decode_expanded_bytes",
    "gqa_decode_plan", "gqa_tp_shard", "gqa_mla_decode", "gqa_mla_decode_cudacore", "gqa_get_last_device_status", "gqa_selftest_wait_timeout", "gqa_set_profile_events",
    "gqa_last_launch_count", "gqa_release", "gqa_set_workspace_allocator", "gqa_status_string", "gqa_version",
    "library_path", "load",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libgqa.so")
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
# gqa_alloc_fn / gqa_free_fn of include/gqa.h
ALLOC_FN = ctypes.CFUNCTYPE(ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p)
FREE_FN = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p)

EXPORTS = {
    # name: (restype, argtypes)
    "gqa_decode": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp]),
    "gqa_decode_fp8": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                            _vp, _vp]),
    "gqa_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp]),
    "gqa_prefill_causal": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "gqa_prefill_causal_fwd": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
    "gqa_prefill_causal_bwd": (_i, [_vp] * 6 + [_i] * 5 + [_vp] * 4),
    "gqa_decode_expanded": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp, _vp, _vp]),
    "gqa_decode_expanded_bytes": (ctypes.c_size_t, [_i, _i, _i, _i]),
    "gqa_decode_plan": (_i, [_i, _i, _i, _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i),
                             ctypes.POINTER(ctypes.c_size_t)]),
    "gqa_tp_shard": (_i, [_i, _i, _i, _i] + [ctypes.POINTER(_i)] * 4),
    "gqa_mla_decode": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp]),
    "gqa_mla_decode_cudacore": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp]),
    "gqa_get_last_device_status": (_i, [_vp]),
    "gqa_selftest_wait_timeout": (_i, [_i, _vp]),
    "gqa_set_profile_events": (_i, [_vp, _vp]),
    "gqa_last_launch_count": (_i, []),
    "gqa_release": (None, []),
    "gqa_set_workspace_allocator": (_i, [_vp, _vp, _vp]),   # ALLOC_FN / FREE_FN pointers or NULL
    "gqa_status_string": (ctypes.c_char_p, [_i]),
    "gqa_version": (ctypes.c_char_p, []),
}


class GQAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_text(status)} (status {status})")


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libgqa.so (built in-tree by ``python -m grouped_query_attention_02_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libgqa.so is not built ({_LIB_PATH}); run "
                               "`python -m grouped_query_attention_02_b200.build` -- there is no fallback path")
        lib = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_text(status: int) -> str:
    return load().gqa_status_string(status).decode()


def _check(status: int, where: str):
    if status != 0:
        raise GQAError(status, where)


def _stream_ptr(stream):
    """The stream argument of an entry point: None = the current device's current stream."""
    import torch

    if stream is None:
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        if raw is not None:   # the handle without building a Stream object (a few microseconds a call)
            return raw(torch._C._cuda_getDevice())
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, ndim, device=None):
    """Checks one tensor argument: type, dtype, rank, a CUDA device (the given one, if any), contiguous.
    The common case costs a handful of attribute reads; the detailed checks run only to name a failure."""
    try:
        if t.dtype is dtype and t.dim() == ndim and t.is_contiguous():
            d = t.get_device()
            if d >= 0 and (device is None or d == (device if isinstance(device, int) else device.index)):
                return
    except AttributeError:
        pass
    import torch

    if isinstance(device, int):
        device = torch.device("cuda", device)
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    raise ValueError(f"{name}: unsupported tensor")


def gqa_decode(q, k_cache, v_cache, seqlens, scale=None, out=None, stream=None):
    """q [B,Hq,d], k_cache/v_cache [B,Tmax,Hkv,d] bf16, seqlens [B] int32 (device) -> out [B,Hq,d] bf16."""
    import torch

    _need(q, "q", torch.bfloat16, 3)
    B, Hq, d = q.shape
    dev = q.get_device()
    _need(k_cache, "k_cache", torch.bfloat16, 4, dev)
    _need(v_cache, "v_cache", torch.bfloat16, 4, dev)
    _need(seqlens, "seqlens", torch.int32, 1, dev)
    Bk, Tmax, Hkv, dk = k_cache.shape
    if (Bk, dk) != (B, d) or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, k_cache, v_cache and seqlens")
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", torch.bfloat16, 3, dev)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    if scale is None:
        scale = 1.0 / d ** 0.5
    st = load().gqa_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(), B, Hq, Hkv, d,
                           Tmax, float(scale), out.data_ptr(), _stream_ptr(stream))
    _check(st, "gqa_decode")
    return out


def gqa_decode_fp8(q, k_cache, v_cache, seqlens, k_scale, v_scale, scale=None, out=None, stream=None):
    """q [B,Hq,d] bf16; k_cache/v_cache [B,Tmax,Hkv,d] E4M3 codes (torch.uint8 or torch.float8_e4m3fn);
    a key is e4m3(code) * k_scale, a value e4m3(code) * v_scale; seqlens [B] int32 (device)
    -> out [B,Hq,d] bf16."""
    import torch

    _need(q, "q", torch.bfloat16, 3)
    B, Hq, d = q.shape
    dev = q.get_device()
    if k_cache.dtype == torch.float8_e4m3fn:
        k_cache = k_cache.view(torch.uint8)
    if v_cache.dtype == torch.float8_e4m3fn:
        v_cache = v_cache.view(torch.uint8)
    _need(k_cache, "k_cache", torch.uint8, 4, dev)
    _need(v_cache, "v_cache", torch.uint8, 4, dev)
    _need(seqlens, "seqlens", torch.int32, 1, dev)
    Bk, Tmax, Hkv, dk = k_cache.shape
    if (Bk, dk) != (B, d) or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, k_cache, v_cache and seqlens")
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", torch.bfloat16, 3, dev)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    if scale is None:
        scale = 1.0 / d ** 0.5
    st = load().gqa_decode_fp8(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(), B, Hq, Hkv,
                               d, Tmax, float(scale), float(k_scale), float(v_scale), out.data_ptr(),
                               _stream_ptr(stream))
    _check(st, "gqa_decode_fp8")
    return out


def gqa_decode_noalloc(q, k_cache, v_cache, seqlens, scale=None, out=None, stream=None):
    """gqa_decode without any device allocation by the library (its split partials live in a fixed
    32 MiB array inside libgqa.so).  For callers whose device memory is fully reserved by their own
    pool, or whose decode loop cannot absorb cudaMalloc.  `out` should be preallocated by such a
    caller; calls that overlap on the GPU race on the shared array."""
    import torch

    _need(q, "q", torch.bfloat16, 3)
    B, Hq, d = q.shape
    _need(k_cache, "k_cache", torch.bfloat16, 4, q.device)
    _need(v_cache, "v_cache", torch.bfloat16, 4, q.device)
    _need(seqlens, "seqlens", torch.int32, 1, q.device)
    Bk, Tmax, Hkv, dk = k_cache.shape
    if (Bk, dk) != (B, d) or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, k_cache, v_cache and seqlens")
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", torch.bfloat16, 3, q.device)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    if scale is None:
        scale = 1.0 / d ** 0.5
    st = load().gqa_decode_noalloc(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(), B, Hq,
                                   Hkv, d, Tmax, float(scale), out.data_ptr(), _stream_ptr(stream))
    _check(st, "gqa_decode_noalloc")
    return out


def gqa_decode_expanded(q, k_cache, v_cache, seqlens, scale=None, out=None, k_rep=None, v_rep=None, stream=None):
    """The repeat-KV baseline: same result as gqa_decode, K/V copied g times first."""
    import torch

    _need(q, "q", torch.bfloat16, 3)
    B, Hq, d = q.shape
    _need(k_cache, "k_cache", torch.bfloat16, 4, q.device)
    _need(v_cache, "v_cache", torch.bfloat16, 4, q.device)
    _need(seqlens, "seqlens", torch.int32, 1, q.device)
    Bk, Tmax, Hkv, dk = k_cache.shape
    if (Bk, dk) != (B, d) or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, k_cache, v_cache and seqlens")
    if out is None:
        out = torch.empty_like(q)
    rep_shape = (B, Tmax, Hq, d)
    if k_rep is None:
        k_rep = torch.empty(rep_shape, dtype=torch.bfloat16, device=q.device)
    if v_rep is None:
        v_rep = torch.empty(rep_shape, dtype=torch.bfloat16, device=q.device)
    for t, n in ((out, "out"), (k_rep, "k_rep"), (v_rep, "v_rep")):
        _need(t, n, torch.bfloat16, t.dim(), q.device)
    if tuple(k_rep.shape) != rep_shape or tuple(v_rep.shape) != rep_shape:
        raise ValueError(f"k_rep/v_rep must have shape {rep_shape}")
    if scale is None:
        scale = 1.0 / d ** 0.5
    st = load().gqa_decode_expanded(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(), B, Hq,
                                    Hkv, d, Tmax, float(scale), out.data_ptr(), k_rep.data_ptr(), v_rep.data_ptr(),
                                    _stream_ptr(stream))
    _check(st, "gqa_decode_expanded")
    return out


def gqa_prefill_causal(q, k, v, out=None, stream=None):
    """q [B,S,Hq,d], k/v [B,S,Hkv,d] bf16 -> out [B,S,Hq,d] bf16 (causal, scale 1/sqrt(d))."""
    import torch

    _need(q, "q", torch.bfloat16, 4)
    B, S, Hq, d = q.shape
    _need(k, "k", torch.bfloat16, 4, q.device)
    _need(v, "v", torch.bfloat16, 4, q.device)
    Bk, Sk, Hkv, dk = k.shape
    if (Bk, Sk, dk) != (B, S, d) or v.shape != k.shape:
        raise ValueError("shape mismatch between q, k and v")
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", torch.bfloat16, 4, q.device)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    st = load().gqa_prefill_causal(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, S, Hq, Hkv, d, out.data_ptr(),
                                   _stream_ptr(stream))
    _check(st, "gqa_prefill_causal")
    return out


def gqa_prefill_causal_fwd(q, k, v, out=None, lse=None, stream=None):
    """gqa_prefill_causal that also returns lse [B,Hq,S] fp32 (natural log-sum-exp of each row's scaled
    scores), for the backward.  Returns (out, lse)."""
    import torch

    _need(q, "q", torch.bfloat16, 4)
    B, S, Hq, d = q.shape
    _need(k, "k", torch.bfloat16, 4, q.device)
    _need(v, "v", torch.bfloat16, 4, q.device)
    Bk, Sk, Hkv, dk = k.shape
    if (Bk, Sk, dk) != (B, S, d) or v.shape != k.shape:
        raise ValueError("shape mismatch between q, k and v")
    out = torch.empty_like(q) if out is None else out
    _need(out, "out", torch.bfloat16, 4, q.device)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(lse, "lse", torch.float32, 3, q.device)
    if out.shape != q.shape or lse.shape != (B, Hq, S):
        raise ValueError("out must have q's shape and lse [B,Hq,S]")
    st = load().gqa_prefill_causal_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, S, Hq, Hkv, d, out.data_ptr(),
                                       lse.data_ptr(), _stream_ptr(stream))
    _check(st, "gqa_prefill_causal_fwd")
    return out, lse


def gqa_prefill_causal_bwd(q, k, v, out, lse, dout, dq=None, dk=None, dv=None, stream=None):
    """Gradients through gqa_prefill_causal: (dq [B,S,Hq,d], dk, dv [B,S,Hkv,d]) bf16; dk and dv are summed
    over each KV head's group of query heads."""
    import torch

    _need(q, "q", torch.bfloat16, 4)
    B, S, Hq, d = q.shape
    _need(k, "k", torch.bfloat16, 4, q.device)
    _need(v, "v", torch.bfloat16, 4, q.device)
    _need(out, "out", torch.bfloat16, 4, q.device)
    _need(dout, "dout", torch.bfloat16, 4, q.device)
    _need(lse, "lse", torch.float32, 3, q.device)
    Hkv = k.shape[2]
    if k.shape != (B, S, Hkv, d) or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape \
            or lse.shape != (B, Hq, S):
        raise ValueError("shape mismatch between q, k, v, out, lse and dout")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, n, torch.bfloat16, 4, q.device)
    if dq.shape != q.shape or dk.shape != k.shape or dv.shape != v.shape:
        raise ValueError("gradient buffers must have the shapes of q, k and v")
    st = load().gqa_prefill_causal_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                       dout.data_ptr(), B, S, Hq, Hkv, d, dq.data_ptr(), dk.data_ptr(),
                                       dv.data_ptr(), _stream_ptr(stream))
    _check(st, "gqa_prefill_causal_bwd")
    return dq, dk, dv


def gqa_decode_expanded_bytes(B, Tmax, Hq, d):
    return int(load().gqa_decode_expanded_bytes(B, Tmax, Hq, d))


def gqa_decode_plan(B, Hq, Hkv, d, Tmax, num_sms):
    """(chunk, nsplit, workspace_bytes) gqa_decode uses on a device with num_sms SMs."""
    c, n, w = _i(), _i(), ctypes.c_size_t()
    _check(load().gqa_decode_plan(B, Hq, Hkv, d, Tmax, num_sms, ctypes.byref(c), ctypes.byref(n), ctypes.byref(w)),
           "gqa_decode_plan")
    return c.value, n.value, w.value


def _mla(fn_name, q, kv_cache, seqlens, scale, out, stream, d_c):
    import torch

    _need(q, "q", torch.bfloat16, 3)
    B, Hq, dk = q.shape
    _need(kv_cache, "kv_cache", torch.bfloat16, 3, q.device)
    _need(seqlens, "seqlens", torch.int32, 1, q.device)
    if kv_cache.shape[0] != B or kv_cache.shape[2] != dk or seqlens.shape[0] != B:
        raise ValueError(f"shapes disagree: q {tuple(q.shape)}, kv_cache {tuple(kv_cache.shape)}, "
                         f"seqlens {tuple(seqlens.shape)}")
    d_r = dk - int(d_c)
    if scale is None:
        scale = 1.0 / float(128 + d_r) ** 0.5
    if out is None:
        out = torch.empty((B, Hq, int(d_c)), dtype=torch.bfloat16, device=q.device)
    else:
        _need(out, "out", torch.bfloat16, 3, q.device)
    _check(getattr(load(), fn_name)(q.data_ptr(), kv_cache.data_ptr(), seqlens.data_ptr(), B, Hq, int(d_c), d_r,
                                    kv_cache.shape[1], ctypes.c_float(scale), out.data_ptr(), _stream_ptr(stream)),
           fn_name)
    return out


def gqa_mla_decode(q, kv_cache, seqlens, scale=None, out=None, stream=None, d_c=512):
    """MLA decode with absorbed weights on the tensor cores: q [B,Hq,d_c+d_r], kv_cache [B,Tmax,d_c+d_r] bf16,
    seqlens [B] int32 (device) -> out [B,Hq,d_c] bf16.  scale defaults to 1/sqrt(128 + d_r)."""
    return _mla("gqa_mla_decode", q, kv_cache, seqlens, scale, out, stream, d_c)


def gqa_mla_decode_cudacore(q, kv_cache, seqlens, scale=None, out=None, stream=None, d_c=512):
    """The same operator on the CUDA cores (fp32 weights): the independent second path for full-size checks."""
    return _mla("gqa_mla_decode_cudacore", q, kv_cache, seqlens, scale, out, stream, d_c)


def gqa_tp_shard(Hq, Hkv, tp, rank):
    """(q_first, q_count, kv_first, kv_count): the query heads and KV heads (partitioned, or one replica when
    Hkv < tp) that rank `rank` of `tp` tensor-parallel ranks owns."""
    a, b, c, d = _i(), _i(), _i(), _i()
    _check(load().gqa_tp_shard(int(Hq), int(Hkv), int(tp), int(rank), ctypes.byref(a), ctypes.byref(b),
                               ctypes.byref(c), ctypes.byref(d)), "gqa_tp_shard")
    return a.value, b.value, c.value, d.value


def gqa_get_last_device_status(stream=None) -> int:
    return int(load().gqa_get_last_device_status(_stream_ptr(stream)))


def gqa_selftest_wait_timeout(timeout_us: int, stream=None):
    _check(load().gqa_selftest_wait_timeout(int(timeout_us), _stream_ptr(stream)), "gqa_selftest_wait_timeout")


def gqa_set_profile_events(before=None, after=None):
    """before/after: torch.cuda.Event(enable_timing=True) or None (turns the hook off)."""
    for ev in (before, after):
        if ev is not None and not ev.cuda_event:
            ev.record()          # torch creates the underlying cudaEvent_t lazily, on first record
    b = None if before is None else ctypes.c_void_p(before.cuda_event)
    a = None if after is None else ctypes.c_void_p(after.cuda_event)
    _check(load().gqa_set_profile_events(b, a), "gqa_set_profile_events")


def gqa_last_launch_count() -> int:
    return int(load().gqa_last_launch_count())


def gqa_release():
    load().gqa_release()


_allocator_refs = None   # the ctypes callbacks the library may call; kept alive while installed


def gqa_set_workspace_allocator(alloc=None, free=None):
    """Take the library's per-device workspace from the caller's pool: ``alloc(nbytes, device)`` returns a
    256-byte aligned device address (0 when there is none), ``free(ptr, nbytes, device)`` takes it back.
    Both None restores cudaMalloc / cudaFree.  Must be called with no library work in flight."""
    global _allocator_refs
    if (alloc is None) != (free is None):
        raise ValueError("alloc and free are installed together")
    if alloc is None:
        _check(load().gqa_set_workspace_allocator(None, None, None), "gqa_set_workspace_allocator")
        _allocator_refs = None   # dropped only now: the call handed the blocks back through them
        return
    ca = ALLOC_FN(lambda nbytes, dev, ctx: int(alloc(int(nbytes), int(dev)) or 0) or None)
    cf = FREE_FN(lambda ptr, nbytes, dev, ctx: free(int(ptr or 0), int(nbytes), int(dev)))
    _check(load().gqa_set_workspace_allocator(ctypes.cast(ca, _vp), ctypes.cast(cf, _vp), None),
           "gqa_set_workspace_allocator")
    _allocator_refs = (ca, cf)


def gqa_status_string(status: int) -> str:
    return status_text(status)


def gqa_version() -> str:
    return load().gqa_version().decode()
