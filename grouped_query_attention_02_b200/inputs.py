"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle leg.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic.  Recipe (the same for every workload):

* q, K, V: i.i.d. N(0, 1) in bf16 (torch normal in fp32, rounded to bf16),
  drawn from ``torch.Generator(device).manual_seed(seed)`` with seeds
  ``base+0`` (q), ``base+1`` (K), ``base+2`` (V);
* seqlens: integers uniform on the closed interval [lo, hi] from seed
  ``base+3`` on a CPU generator (so every device sees the same lengths);
* cache rows at or past ``seqlens[b]`` hold random values too, or NaN when
  ``poison=True`` (a read past the end then shows up as NaN in the output);
* ``q_gain`` multiplies q before rounding (a "peaky" softmax when > 1);
* the backward's incoming gradient dO: N(0, 1) in bf16 from seed ``base+4``.

FP8 caches (``make_decode_fp8``): the same N(0, 1) draws divided by a
per-tensor scale, clamped to the largest finite E4M3 value (448) and stored as
E4M3 codes (torch's float8_e4m3fn cast, round to nearest even); rows past the
history hold the NaN code 0x7F when ``poison=True``.

MLA decode (``make_mla_decode``): q [B,Hq,d_c+d_r] (absorbed latent query, then
RoPE query) from seed ``base+0`` and the cache [B,Tmax,d_c+d_r] (latent, then the
shared RoPE key) from seed ``base+1``, both N(0, 1) bf16; the default scale is
1/sqrt(d_h + d_r) with the original per-head width d_h = 128.

Layouts are the ones of the C ABI: decode q [B,Hq,d], caches [B,Tmax,Hkv,d];
prefill q [B,S,Hq,d], k/v [B,S,Hkv,d].
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


def _normal(shape, seed: int, device, gain: float = 1.0) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.empty(shape, dtype=torch.float32, device=device)
    # fill in slices so a 34 GB cache never needs a 68 GB fp32 temporary
    flat = x.view(-1)
    step = 1 << 28
    for s in range(0, flat.numel(), step):
        flat[s:s + step].normal_(generator=g)
    if gain != 1.0:
        x.mul_(gain)
    return x.to(torch.bfloat16)


def _normal_bf16(shape, seed: int, device) -> torch.Tensor:
    """N(0,1) bf16 drawn in slices straight into a bf16 buffer (large caches)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    step = 1 << 27
    tmp = torch.empty(min(step, max(flat.numel(), 1)), dtype=torch.float32, device=device)
    for s in range(0, flat.numel(), step):
        n = min(step, flat.numel() - s)
        t = tmp[:n]
        t.normal_(generator=g)
        flat[s:s + n].copy_(t)
    return out


def seqlens_uniform(B: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """B integers uniform on [lo, hi] (inclusive), CPU int32."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


@dataclass
class DecodeInputs:
    q: torch.Tensor          # [B,Hq,d] bf16
    k_cache: torch.Tensor    # [B,Tmax,Hkv,d] bf16
    v_cache: torch.Tensor    # [B,Tmax,Hkv,d] bf16
    seqlens: torch.Tensor    # [B] int32, same device as q
    scale: float


def make_decode(B: int, Hq: int, Hkv: int, d: int, Tmax: int, seqlens=None, *, device="cpu",
                seed: int = 0, scale: float | None = None, poison: bool = False,
                q_gain: float = 1.0, seqlen_range=None) -> DecodeInputs:
    """Decode inputs.  ``seqlens``: None -> every sequence holds Tmax tokens;
    an int -> all equal; a list/tensor -> as given; or ``seqlen_range=(lo,hi)``
    draws them uniformly with seed ``seed+3``."""
    if seqlen_range is not None:
        sl = seqlens_uniform(B, seqlen_range[0], seqlen_range[1], seed + 3)
    elif seqlens is None:
        sl = torch.full((B,), Tmax, dtype=torch.int32)
    elif isinstance(seqlens, int):
        sl = torch.full((B,), seqlens, dtype=torch.int32)
    else:
        sl = torch.as_tensor(seqlens, dtype=torch.int32).cpu()
    q = _normal((B, Hq, d), seed + 0, device, q_gain)
    big = B * Tmax * Hkv * d > (1 << 26)
    mk = _normal_bf16 if big else _normal
    k = mk((B, Tmax, Hkv, d), seed + 1, device)
    v = mk((B, Tmax, Hkv, d), seed + 2, device)
    if poison:
        nan = torch.tensor(float("nan"), dtype=torch.bfloat16, device=device)
        for b in range(B):
            t = int(sl[b])
            if t < Tmax:
                k[b, t:].fill_(nan)
                v[b, t:].fill_(nan)
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    return DecodeInputs(q, k, v, sl.to(device), scale)


@dataclass
class DecodeFp8Inputs:
    q: torch.Tensor          # [B,Hq,d] bf16
    k_cache: torch.Tensor    # [B,Tmax,Hkv,d] uint8, E4M3 codes
    v_cache: torch.Tensor    # [B,Tmax,Hkv,d] uint8, E4M3 codes
    k_scale: float           # a key is e4m3(code) * k_scale
    v_scale: float           # a value is e4m3(code) * v_scale
    seqlens: torch.Tensor    # [B] int32, same device as q
    scale: float


def _normal_e4m3(shape, seed: int, device, inv_scale: float) -> torch.Tensor:
    """N(0,1) / scale, clamped to +-448 and cast to E4M3 codes, drawn in slices."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    flat = out.view(-1)
    step = 1 << 27
    tmp = torch.empty(min(step, max(flat.numel(), 1)), dtype=torch.float32, device=device)
    for s in range(0, flat.numel(), step):
        n = min(step, flat.numel() - s)
        t = tmp[:n]
        t.normal_(generator=g)
        t.mul_(inv_scale).clamp_(-448.0, 448.0)
        flat[s:s + n].copy_(t.to(torch.float8_e4m3fn).view(torch.uint8))
    return out


def make_decode_fp8(B: int, Hq: int, Hkv: int, d: int, Tmax: int, seqlens=None, *, device="cpu",
                    seed: int = 0, scale: float | None = None, poison: bool = False, q_gain: float = 1.0,
                    seqlen_range=None, k_scale: float = 0.0135, v_scale: float = 0.0142) -> DecodeFp8Inputs:
    """Decode inputs over an FP8 (E4M3) cache with per-tensor scales; ``seqlens`` as in make_decode.
    The default scales map about six standard deviations onto the largest E4M3 value.  The codes are
    N(0,1) / scale; a zero scale draws them with the default scale (its keys or values are all zero)."""
    if seqlen_range is not None:
        sl = seqlens_uniform(B, seqlen_range[0], seqlen_range[1], seed + 3)
    elif seqlens is None:
        sl = torch.full((B,), Tmax, dtype=torch.int32)
    elif isinstance(seqlens, int):
        sl = torch.full((B,), seqlens, dtype=torch.int32)
    else:
        sl = torch.as_tensor(seqlens, dtype=torch.int32).cpu()
    q = _normal((B, Hq, d), seed + 0, device, q_gain)
    k = _normal_e4m3((B, Tmax, Hkv, d), seed + 1, device, 1.0 / (k_scale or 0.0135))
    v = _normal_e4m3((B, Tmax, Hkv, d), seed + 2, device, 1.0 / (v_scale or 0.0142))
    if poison:
        for b in range(B):
            t = int(sl[b])
            if t < Tmax:
                k[b, t:].fill_(0x7F)
                v[b, t:].fill_(0x7F)
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    return DecodeFp8Inputs(q, k, v, float(k_scale), float(v_scale), sl.to(device), scale)


@dataclass
class PrefillInputs:
    q: torch.Tensor   # [B,S,Hq,d] bf16
    k: torch.Tensor   # [B,S,Hkv,d] bf16
    v: torch.Tensor   # [B,S,Hkv,d] bf16
    scale: float


def make_prefill(B: int, S: int, Hq: int, Hkv: int, d: int, *, device="cpu", seed: int = 0,
                 q_gain: float = 1.0) -> PrefillInputs:
    q = _normal((B, S, Hq, d), seed + 0, device, q_gain)
    k = _normal((B, S, Hkv, d), seed + 1, device)
    v = _normal((B, S, Hkv, d), seed + 2, device)
    return PrefillInputs(q, k, v, 1.0 / float(d) ** 0.5)


def make_dout(B: int, S: int, Hq: int, d: int, *, device="cpu", seed: int = 0) -> torch.Tensor:
    """Incoming gradient dO [B,S,Hq,d] of the causal prefill's output (seed ``seed+4``)."""
    return _normal((B, S, Hq, d), seed + 4, device)


@dataclass
class MlaDecodeInputs:
    q: torch.Tensor          # [B,Hq,d_c+d_r] bf16: absorbed latent query, then RoPE query
    kv_cache: torch.Tensor   # [B,Tmax,d_c+d_r] bf16: latent, then the RoPE key shared by all heads
    seqlens: torch.Tensor    # [B] int32, same device as q
    d_c: int
    scale: float


def make_mla_decode(B: int, Hq: int, Tmax: int, d_c: int = 512, d_r: int = 64, seqlens=None, *, device="cpu",
                    seed: int = 0, scale: float | None = None, q_gain: float = 1.0, seqlen_range=None,
                    d_h: int = 128) -> MlaDecodeInputs:
    """MLA decode inputs; ``seqlens`` as in make_decode.  The default scale is 1/sqrt(d_h + d_r)."""
    if seqlen_range is not None:
        sl = seqlens_uniform(B, seqlen_range[0], seqlen_range[1], seed + 3)
    elif seqlens is None:
        sl = torch.full((B,), Tmax, dtype=torch.int32)
    elif isinstance(seqlens, int):
        sl = torch.full((B,), seqlens, dtype=torch.int32)
    else:
        sl = torch.as_tensor(seqlens, dtype=torch.int32).cpu()
    dk = d_c + d_r
    q = _normal((B, Hq, dk), seed + 0, device, q_gain)
    mk = _normal_bf16 if B * Tmax * dk > (1 << 26) else _normal
    kv = mk((B, Tmax, dk), seed + 1, device)
    if scale is None:
        scale = 1.0 / float(d_h + d_r) ** 0.5
    return MlaDecodeInputs(q, kv, sl.to(device), d_c, scale)

