"""fp64 CPU oracle for grouped-query attention (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding in ``grouped_query_attention_02_b200``) never touches it, and the
two share no code.

The arithmetic lives in ``gqa_oracle.c`` (plain C, double precision, explicit
per-head K/V repeat, two-pass softmax); this module only marshals arguments
through ctypes.  Pages it follows:

* mapping and regular grouping: study.greatitself.com "grouped-query and
  multi-query attention", the mapping paragraph; lihaoran.work/?p=2890
  "Shared KV can still produce different outputs" (8 -> 2 mapping check);
* KV bytes: lihaoran.work/?p=2890 "KV-head count determines the raw cache
  ratio";
* per-head attention and the causal mask: anrans.github.io attention-variants,
  "Kernels do not need to copy the KV heads" (the expanded version);
* MLA decode with absorbed weights: anrans.github.io attention-variants,
  "MLA: multi-head latent attention" (weight absorption, decoupled RoPE).

Every function is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_LIB = os.path.join(_HERE, "libgqa_oracle.so")


def compile_oracle(src: str, lib: str) -> str:
    """gcc -O2 with pthreads; used for the oracle itself and for the planted-mistake tests."""
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", lib, src, "-lm"])
    return lib


def build(force: bool = False) -> str:
    """Compile the oracle next to its source when missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_oracle(_SRC, _LIB)
    return _LIB


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _bits(x) -> np.ndarray:
    """bf16 tensor (torch, any device) or uint16 array -> contiguous uint16 numpy."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch

    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _bytes(x) -> np.ndarray:
    """FP8 tensor (torch float8_e4m3fn or uint8, any device) or uint8 array -> contiguous uint8 numpy."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint8
        return np.ascontiguousarray(x)
    import torch

    t = x.detach().cpu().contiguous()
    if t.dtype != torch.uint8:
        t = t.view(torch.uint8)
    return np.ascontiguousarray(t.numpy())


class Oracle:
    """ctypes view of one compiled copy of gqa_oracle.c."""

    def __init__(self, libpath: str):
        lib = ctypes.CDLL(libpath)
        lib.gqa_oracle_kv_head.restype = ctypes.c_int
        lib.gqa_oracle_kv_head.argtypes = [ctypes.c_int] * 3
        lib.gqa_oracle_kv_bytes.restype = ctypes.c_longlong
        lib.gqa_oracle_kv_bytes.argtypes = [ctypes.c_longlong] * 5
        lib.gqa_oracle_bf16_to_f64.restype = None
        lib.gqa_oracle_bf16_to_f64.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong]
        lib.gqa_oracle_decode.restype = ctypes.c_int
        lib.gqa_oracle_decode.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 5 + [
            ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
        lib.gqa_oracle_prefill_backward.restype = ctypes.c_int
        lib.gqa_oracle_prefill_backward.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 5 + [
            ctypes.c_double] + [ctypes.c_void_p] * 5 + [ctypes.c_int]
        lib.gqa_oracle_e4m3_to_f64.restype = None
        lib.gqa_oracle_e4m3_to_f64.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong]
        lib.gqa_oracle_decode_fp8.restype = ctypes.c_int
        lib.gqa_oracle_decode_fp8.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_double] * 2 + [ctypes.c_void_p] + [
            ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
        lib.gqa_oracle_mla_decode.restype = ctypes.c_int
        lib.gqa_oracle_mla_decode.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [
            ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
        lib.gqa_oracle_prefill.restype = ctypes.c_int
        lib.gqa_oracle_prefill.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [
            ctypes.c_double, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p, ctypes.c_int]
        self.lib = lib

    def kv_head(self, h: int, Hq: int, Hkv: int) -> int:
        return self.lib.gqa_oracle_kv_head(h, Hq, Hkv)

    def kv_bytes(self, layers: int, tokens: int, kv_heads: int, head_dim: int, bytes_per_elem: int) -> int:
        return self.lib.gqa_oracle_kv_bytes(layers, tokens, kv_heads, head_dim, bytes_per_elem)

    def bf16_bits_to_f64(self, bits: np.ndarray) -> np.ndarray:
        b = np.ascontiguousarray(bits, dtype=np.uint16)
        out = np.empty(b.shape, dtype=np.float64)
        self.lib.gqa_oracle_bf16_to_f64(b.ctypes.data, out.ctypes.data, b.size)
        return out

    def prefill_backward(self, q, k, v, dout, scale: float, row_sel=None, key_sel=None,
                         nthreads: int | None = None):
        """Causal prefill backward: q, dout [B,S,Hq,d], k, v [B,S,Hkv,d] (bf16) -> (dq, dk, dv) fp64.
        row_sel / key_sel: optional iterables of positions whose dq / dk, dv are computed (others 0)."""
        qb, kb, vb, ob = _bits(q), _bits(k), _bits(v), _bits(dout)
        B, S, Hq, d = qb.shape
        Hkv = kb.shape[2]
        assert kb.shape == (B, S, Hkv, d) and vb.shape == kb.shape and ob.shape == qb.shape

        def flags(sel):
            if sel is None:
                return None
            f = np.zeros(S, dtype=np.int32)
            f[np.asarray(list(sel), dtype=np.int64)] = 1
            return f

        rf, kf = flags(row_sel), flags(key_sel)
        dq = np.empty((B, S, Hq, d), dtype=np.float64)
        dk = np.empty((B, S, Hkv, d), dtype=np.float64)
        dv = np.empty((B, S, Hkv, d), dtype=np.float64)
        st = self.lib.gqa_oracle_prefill_backward(
            qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, ob.ctypes.data, B, S, Hq, Hkv, d, float(scale),
            None if rf is None else rf.ctypes.data, None if kf is None else kf.ctypes.data,
            dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, nthreads or default_threads())
        if st != 0:
            raise ValueError(f"oracle backward rejected its arguments (status {st})")
        return dq, dk, dv

    def e4m3_to_f64(self, bytes_: np.ndarray) -> np.ndarray:
        b = np.ascontiguousarray(bytes_, dtype=np.uint8)
        out = np.empty(b.shape, dtype=np.float64)
        self.lib.gqa_oracle_e4m3_to_f64(b.ctypes.data, out.ctypes.data, b.size)
        return out

    def decode_fp8(self, q, k8, v8, k_scale: float, v_scale: float, seqlens, scale: float,
                   nthreads: int | None = None) -> np.ndarray:
        """q [B,Hq,d] bf16; k8/v8 [B,Tmax,Hkv,d] E4M3 bytes (uint8 or float8_e4m3fn) -> out fp64."""
        qb, kb, vb = _bits(q), _bytes(k8), _bytes(v8)
        B, Hq, d = qb.shape
        B2, Tmax, Hkv, d2 = kb.shape
        assert B2 == B and d2 == d and vb.shape == kb.shape
        sl = np.ascontiguousarray(np.asarray(
            seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int32))
        out = np.zeros((B, Hq, d), dtype=np.float64)
        st = self.lib.gqa_oracle_decode_fp8(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, float(k_scale),
                                            float(v_scale), sl.ctypes.data, B, Hq, Hkv, d, Tmax, float(scale),
                                            out.ctypes.data, nthreads or default_threads())
        if st != 0:
            raise ValueError(f"oracle fp8 decode rejected its arguments (status {st})")
        return out

    def decode(self, q, k_cache, v_cache, seqlens, scale: float, nthreads: int | None = None) -> np.ndarray:
        """q [B,Hq,d], k/v [B,Tmax,Hkv,d] (bf16), seqlens [B] -> out [B,Hq,d] fp64."""
        qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
        B, Hq, d = qb.shape
        B2, Tmax, Hkv, d2 = kb.shape
        assert B2 == B and d2 == d and vb.shape == kb.shape
        sl = np.ascontiguousarray(np.asarray(
            seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int32))
        assert sl.shape == (B,)
        out = np.zeros((B, Hq, d), dtype=np.float64)
        st = self.lib.gqa_oracle_decode(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, sl.ctypes.data,
                                        B, Hq, Hkv, d, Tmax, float(scale), out.ctypes.data,
                                        nthreads or default_threads())
        if st != 0:
            raise ValueError(f"oracle decode rejected its arguments (status {st})")
        return out

    def mla_decode(self, q, kv, seqlens, d_c: int, scale: float, nthreads: int | None = None) -> np.ndarray:
        """MLA decode with absorbed weights: q [B,Hq,d_c+d_r], kv [B,Tmax,d_c+d_r] (bf16; latent then RoPE
        part), seqlens [B] -> out [B,Hq,d_c] fp64, the softmax-weighted sum of the rows' latent parts."""
        qb, kb = _bits(q), _bits(kv)
        B, Hq, dk = qb.shape
        B2, Tmax, dk2 = kb.shape
        assert B2 == B and dk2 == dk and 0 < d_c <= dk
        sl = np.ascontiguousarray(np.asarray(
            seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int32))
        assert sl.shape == (B,)
        out = np.zeros((B, Hq, d_c), dtype=np.float64)
        st = self.lib.gqa_oracle_mla_decode(qb.ctypes.data, kb.ctypes.data, sl.ctypes.data, B, Hq, d_c, dk - d_c,
                                            Tmax, float(scale), out.ctypes.data, nthreads or default_threads())
        if st != 0:
            raise ValueError(f"oracle MLA decode rejected its arguments (status {st})")
        return out

    def prefill_causal(self, q, k, v, scale: float, rows=None, nthreads: int | None = None) -> np.ndarray:
        """q [B,S,Hq,d], k/v [B,S,Hkv,d] (bf16).

        rows None -> out [B,S,Hq,d] fp64.  rows = int array [n,3] of (b, h, r)
        -> out [n,d] fp64, those rows in the given order."""
        qb, kb, vb = _bits(q), _bits(k), _bits(v)
        B, S, Hq, d = qb.shape
        B2, S2, Hkv, d2 = kb.shape
        assert (B2, S2, d2) == (B, S, d) and vb.shape == kb.shape
        if rows is None:
            out = np.zeros((B, S, Hq, d), dtype=np.float64)
            r, rp, n = None, None, 0
        else:
            r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
            out = np.zeros((r.shape[0], d), dtype=np.float64)
            rp, n = r.ctypes.data, r.shape[0]
        st = self.lib.gqa_oracle_prefill(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, B, S, Hq, Hkv, d,
                                         float(scale), rp, n, out.ctypes.data,
                                         nthreads or default_threads())
        if st != 0:
            raise ValueError(f"oracle prefill rejected its arguments (status {st})")
        return out


_default = None


def _get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def kv_head(h, Hq, Hkv):
    return _get().kv_head(h, Hq, Hkv)


def kv_bytes(layers, tokens, kv_heads, head_dim, bytes_per_elem):
    return _get().kv_bytes(layers, tokens, kv_heads, head_dim, bytes_per_elem)


def bf16_bits_to_f64(bits):
    return _get().bf16_bits_to_f64(bits)


def decode(q, k_cache, v_cache, seqlens, scale, nthreads=None):
    return _get().decode(q, k_cache, v_cache, seqlens, scale, nthreads)


def e4m3_to_f64(bytes_):
    return _get().e4m3_to_f64(bytes_)


def prefill_backward(q, k, v, dout, scale, row_sel=None, key_sel=None, nthreads=None):
    return _get().prefill_backward(q, k, v, dout, scale, row_sel, key_sel, nthreads)


def decode_fp8(q, k8, v8, k_scale, v_scale, seqlens, scale, nthreads=None):
    return _get().decode_fp8(q, k8, v8, k_scale, v_scale, seqlens, scale, nthreads)


def mla_decode(q, kv, seqlens, d_c, scale, nthreads=None):
    return _get().mla_decode(q, kv, seqlens, d_c, scale, nthreads)


def prefill_causal(q, k, v, scale, rows=None, nthreads=None):
    return _get().prefill_causal(q, k, v, scale, rows, nthreads)
