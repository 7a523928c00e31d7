"""Planted mistakes: each plausible slip in the oracle must break at least one pin.

Every case copies ``oracle/gqa_oracle.c`` to a temporary directory, changes
one fragment (a dropped term, a wrong index, a strided mapping, an off-by-one
in the causal mask ...), compiles it with gcc and runs the pin suite of
``test_oracle_pins`` against that copy.  The oracle source itself is never
modified.  CPU only.
"""
from __future__ import annotations

import inspect
import os

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gqa_oracle.c")

MUTANTS = {
    "strided mapping": ("return h / group;", "return h % Hkv;"),
    "dropped scale": ("s *= scale;", "s *= 1.0;"),
    "causal mask excludes the diagonal": ("attend_row(qrow, Kh, Vh, r + 1,", "attend_row(qrow, Kh, Vh, r,"),
    "no normalisation": ("out[j] /= denom;", "out[j] /= 1.0;"),
    "values read from the key cache": ("Vh[t * d + j] = bf16_to_double(J->v[src + j]);",
                                       "Vh[t * d + j] = bf16_to_double(J->k[src + j]);"),
    "cache read as [B,Hkv,T,d]": (
        "size_t src = (((size_t)b * J->Tmax + (size_t)t) * J->Hkv + (size_t)kvh) * (size_t)d;",
        "size_t src = (((size_t)b * J->Hkv + (size_t)kvh) * J->Tmax + (size_t)t) * (size_t)d;"),
    "query row index transposed": ("size_t qo = ((size_t)b * J->Hq + (size_t)h) * (size_t)d;",
                                   "size_t qo = ((size_t)h * J->B + (size_t)b) * (size_t)d;"),
    "decode drops the newest token": ("attend_row(qrow, Kh, Vh, T, d,", "attend_row(qrow, Kh, Vh, T - 1, d,"),
    "bf16 widening shifted wrong": ("((uint32_t)bits) << 16", "((uint32_t)bits) << 15"),
    "kv bytes count K only": ("return 2LL * layers", "return 1LL * layers"),
    "softmax without exponent": ("double w = exp(scores[t] - m);", "double w = scores[t] - m + 1.0;"),
    "prefill key cache indexed with S and Hq": (
        "size_t src = (((size_t)b * S + (size_t)t) * J->Hkv + (size_t)kvh) * (size_t)d;",
        "size_t src = (((size_t)b * S + (size_t)t) * J->Hq + (size_t)kvh) * (size_t)d;"),
    "e4m3 exponent bias 8": ("else v = ldexp(1.0 + m / 8.0, e - 7);", "else v = ldexp(1.0 + m / 8.0, e - 8);"),
    "e4m3 subnormals one binade low": ("if (e == 0) v = ldexp((double)m, -9);",
                                       "if (e == 0) v = ldexp((double)m, -10);"),
    "e4m3 NaN code read as a number": ("if (e == 15 && m == 7) return NAN;", "if (e == 16) return NAN;"),
    "fp8 key scale dropped": ("Kh[t * d + j] = e4m3_to_double(J->k8[src + j]) * J->k_scale;",
                              "Kh[t * d + j] = e4m3_to_double(J->k8[src + j]);"),
    "backward drops the D term": ("const double dS = P * (dP - Dr[r]);\n                    for (int j = 0; j < d; ++j) dq[j]",
                                  "const double dS = P * dP;\n                    for (int j = 0; j < d; ++j) dq[j]"),
    "backward dk without scale": ("dk[j] += J->scale * dS * Qh[(size_t)r * d + j];", "dk[j] += dS * Qh[(size_t)r * d + j];"),
    "backward dv weighted by dS": ("dv[j] += P * dOh[(size_t)r * d + j];", "dv[j] += dS * dOh[(size_t)r * d + j];"),
    "backward keys skip their own row": ("for (int r = t; r < S; ++r) {", "for (int r = t + 1; r < S; ++r) {"),
    "backward group gradient from one head": ("if (J->key_sel && !J->key_sel[t]) continue;",
                                              "if ((J->key_sel && !J->key_sel[t]) || hh > 0) continue;"),
    "MLA value read from the RoPE end of the row": ("for (int j = 0; j < dv; ++j) Vh[t * dv + j] = bf16_to_double(row[j]);",
                                                   "for (int j = 0; j < dv; ++j) Vh[t * dv + j] = bf16_to_double(row[j + J->dr]);"),
    "MLA scores drop the RoPE part": ("for (int i = 0; i < dk; ++i) s += qrow[i] * Kh[t * dk + i];",
                                      "for (int i = 0; i < dv; ++i) s += qrow[i] * Kh[t * dk + i];"),
    "MLA scale left out": ("w[t] = s * J->scale;", "w[t] = s;"),
    "MLA every head reads head 0's query": (
        "const uint16_t *qs = J->q + ((size_t)b * J->Hq + (size_t)h) * (size_t)dk;",
        "const uint16_t *qs = J->q + ((size_t)b * J->Hq) * (size_t)dk;"),
    "MLA cache rows strided by the value width": (
        "const uint16_t *row = J->kv + ((size_t)b * J->Tmax + (size_t)t) * (size_t)dk;",
        "const uint16_t *row = J->kv + ((size_t)b * J->Tmax + (size_t)t) * (size_t)dv;"),
    "fp8 values scaled by the key scale": ("Vh[t * d + j] = e4m3_to_double(J->v8[src + j]) * J->v_scale;",
                                           "Vh[t * d + j] = e4m3_to_double(J->v8[src + j]) * J->k_scale;"),
}


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if name.startswith("test_"):
            out.append((name, fn))
    return out


def _run_pins(mut):
    failed = []
    for name, fn in _pin_functions():
        params = inspect.signature(fn).parameters
        kwargs = {"oracle_mod": mut}
        if "Hq" in params:
            kwargs.update(Hq=12, Hkv=3)
        if "d" in params:
            kwargs["d"] = 16
        try:
            fn(**kwargs)
        except Exception:  # a failed assertion, a rejected argument, or a crash of the mutant's checks
            failed.append(name)
    return failed


def test_unmodified_copy_passes_every_pin(tmp_path):
    lib = oracle.compile_oracle(SRC, str(tmp_path / "liborig.so"))
    assert _run_pins(oracle.Oracle(lib)) == []


@pytest.mark.parametrize("label", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, label):
    old, new = MUTANTS[label]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"fragment for '{label}' not found in the oracle source"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = oracle.compile_oracle(str(src), str(tmp_path / "libmutant.so"))
    failed = _run_pins(oracle.Oracle(lib))
    assert failed, f"no pin caught the planted mistake '{label}'"
