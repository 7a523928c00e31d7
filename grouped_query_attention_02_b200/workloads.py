"""The five synthetic workloads, by what they are and their sizes.

Shapes follow the pages: the 32/8/128 head geometry read off a config file in
deepconcepts.dev "Checking it on a real system", the 32-query / 2-KV-head
geometry of inferencex.semianalysis.com "Engineering details" (KV head
replication), and the causal prefill of anrans.github.io attention-variants.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    Tmax: int
    seqlen_range: tuple | None = None   # None: every sequence holds Tmax tokens

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    d: int


TINY_DECODE = DecodeWorkload("tiny decode B1 Hq8 Hkv2 d128 T256", 1, 8, 2, 128, 256)
QWEN3_8B_DECODE = DecodeWorkload("Qwen3-8B-shaped decode B49 Hq32 Hkv8 d128 T8192", 49, 32, 8, 128, 8192)
VARLEN_DECODE = tuple(
    DecodeWorkload(f"variable-length decode B64 Hq32 Hkv{h} d128 T~U[512,32768]", 64, 32, h, 128, 32768,
                   (512, 32768))
    for h in (32, 8, 4, 1)
)
EXTREME_GROUP_DECODE = DecodeWorkload(
    "extreme grouping decode (Qwen3.5-style, 32 q heads / 2 KV heads) B16 d128 T131072", 16, 32, 2, 128, 131072)
CAUSAL_PREFILL = PrefillWorkload("causal GQA prefill B4 S8192 Hq32 Hkv8 d128", 4, 8192, 32, 8, 128)

DECODE_WORKLOADS = (TINY_DECODE, QWEN3_8B_DECODE) + VARLEN_DECODE + (EXTREME_GROUP_DECODE,)


@dataclass(frozen=True)
class MlaWorkload:
    name: str
    B: int
    Hq: int
    d_c: int
    d_r: int
    Tmax: int


# MLA decode with absorbed weights in DeepSeek-V3's geometry as the MLA page gives it (128 query heads,
# a 512-wide latent plus a 64-wide RoPE key per token); the page gives no batch or length, so 32
# sequences of 8192 tokens (a 302 MB cache, larger than L2) stand in.
MLA_DECODE = MlaWorkload("MLA absorbed decode (DeepSeek-V3-shaped) B32 Hq128 d_c512 d_r64 T8192", 32, 128, 512, 64,
                         8192)
