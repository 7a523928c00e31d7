"""The MLA decode kernel's decomposition, replayed on the CPU in float64 (no GPU).

`csrc/mla.cu` splits the work into token ranges (its host plan), 16-head blocks and
32-row tiles, keeps a base-2 running maximum and weight sum per head, assigns each
thread one head and 32 latent coordinates, and merges the ranges with weights
2^(m_s - M).  This test replays exactly that order of work in float64 and checks
that it reproduces the fp64 oracle, writes every output once, and never reads a
cached row at or past a sequence's length.
"""
from __future__ import annotations

import numpy as np
import pytest

from grouped_query_attention_02_b200 import inputs

LATENT, ROW, HEADS, TILE = 512, 576, 16, 32


def _plan(B, Hq, Tmax, sms):
    blocks = B * ((Hq + HEADS - 1) // HEADS)
    want = (2 * sms + blocks - 1) // blocks
    nsplit = max(1, min(want, (Tmax + 255) // 256))
    chunk = (Tmax + nsplit - 1) // nsplit
    chunk = (chunk + TILE - 1) // TILE * TILE
    return (Tmax + chunk - 1) // chunk, chunk


def _replay(x, sms):
    q = x.q.double().numpy()
    kv = x.kv_cache.double().numpy()
    B, Hq, _ = q.shape
    Tmax = kv.shape[1]
    nsplit, chunk = _plan(B, Hq, Tmax, sms)
    qscale = x.scale / np.log(2.0)
    out = np.zeros((B, Hq, LATENT))
    writes = np.zeros((B, Hq), dtype=int)
    part = {}
    for b in range(B):
        T = min(max(int(x.seqlens[b]), 0), Tmax)
        for h0 in range(0, Hq, HEADS):
            nh = min(HEADS, Hq - h0)
            qs = np.zeros((HEADS, ROW))
            qs[:nh] = q[b, h0:h0 + nh] * qscale
            for split in range(nsplit):
                tb, te = split * chunk, min(split * chunk + chunk, T)
                m = np.full(HEADS, -np.inf)
                l = np.zeros(HEADS)
                o = np.zeros((HEADS, LATENT))
                for t0 in range(tb, te, TILE):
                    n = min(TILE, te - t0)
                    assert t0 + n <= T                      # no row at or past the history is read
                    rows = kv[b, t0:t0 + n]
                    s = qs @ rows.T                          # [16, n] scores in log2 units
                    m_new = np.maximum(m, s.max(axis=1))
                    alpha = np.where(m == -np.inf, 0.0, np.exp2(m - m_new))
                    p = np.exp2(s - m_new[:, None])
                    l = l * alpha + p.sum(axis=1)
                    o = o * alpha[:, None] + p @ rows[:, :LATENT]
                    m = m_new
                for hh in range(nh):
                    if nsplit == 1:
                        out[b, h0 + hh] = o[hh] / l[hh] if l[hh] != 0 else 0.0
                        writes[b, h0 + hh] += 1
                    else:
                        part[(b, h0 + hh, split)] = (o[hh], m[hh], l[hh])
    if nsplit > 1:
        for b in range(B):
            for h in range(Hq):
                ms = np.array([part[(b, h, s)][1] for s in range(nsplit)])
                M = ms.max()
                w = np.where(ms == -np.inf, 0.0, np.exp2(ms - M))
                L = sum(part[(b, h, s)][2] * w[s] for s in range(nsplit))
                O = sum(part[(b, h, s)][0] * w[s] for s in range(nsplit))
                out[b, h] = O / L if L != 0 else 0.0
                writes[b, h] += 1
    assert np.all(writes == 1)
    return out, nsplit


@pytest.mark.parametrize("B,Hq,Tmax,lens,sms", [
    (2, 20, 70, [70, 0], 148),      # one range; a ragged head block; an empty history
    (1, 16, 600, [600], 148),       # several ranges merged
    (3, 5, 300, [300, 33, 1], 4),   # few SMs; lengths at and off tile edges
    (2, 33, 100, [99, 64], 1),      # one SM: one range per sequence
])
def test_mla_decomposition_reproduces_the_oracle(oracle_mod, B, Hq, Tmax, lens, sms):
    x = inputs.make_mla_decode(B, Hq, Tmax, seqlens=lens, seed=7)
    got, nsplit = _replay(x, sms)
    assert (nsplit > 1) == (B == 1 or sms == 4)
    ref = oracle_mod.mla_decode(x.q, x.kv_cache, x.seqlens, 512, x.scale)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)
