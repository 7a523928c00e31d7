"""Benchmark: GQA decode on one B200 (or N independent GPUs), through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--rows all|none]

One step is one decode step (split-KV kernel + combine) over the Qwen3-8B-shaped
workload: 49 sequences, 32 query heads / 8 KV heads, d=128, 8192 cached tokens
each, bf16 N(0,1) synthetic inputs already resident in HBM.  The cache
(1.64 GB) is larger than the 126 MB L2, so no flush is needed between steps.
The headline value is unique-KV bytes (2 * sum(T) * Hkv * d * 2) per second;
tokens/s (sequences decoded per second, one layer) rides along.

The JSON line also carries the other hot-path rows measured the same way
(tiny decode, variable-length sweep, extreme grouping, the expanded repeat-KV
baseline, FP8 (E4M3) caches of the headline, two variable-length and the
extreme-grouping shapes, causal prefill), the roofline of the dominant kernel, the clocks
seen during the timed region, an end-to-end figure with host buffers, and the
fp64 CPU oracle timed on a bounded sample of the same workload.

With N > 1 (torchrun), every rank decodes its own 49 sequences (its shard of
a 49*N batch; weak scaling, no collective on the data path); the step time is
the maximum over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
PROFILES = os.path.join(ROOT, "profiles")
METRIC = "GQA decode unique-KV HBM GB/s (% of B200 peak) and decode tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- host helpers (no GPU needed)

def unique_kv_bytes(seqlens, Hkv: int, d: int, elem_bytes: int = 2) -> int:
    """K and V rows actually cached: 2 * sum(T) * Hkv * d * elem_bytes (2 for bf16, 1 for FP8)."""
    return 2 * int(sum(int(t) for t in seqlens)) * Hkv * d * elem_bytes


def decode_flops(seqlens, Hq: int, d: int) -> int:
    """4 * Hq * d per cached token: q.k and p.v, independent of Hkv."""
    return 4 * int(sum(int(t) for t in seqlens)) * Hq * d


def prefill_causal_flops(B: int, S: int, Hq: int, d: int) -> int:
    """4 * d per unmasked (query, key) pair per head; row r sees r + 1 keys."""
    return 4 * d * B * Hq * S * (S + 1) // 2


def rank_seed(rank: int, base: int = 0) -> int:
    return base + 1000 * rank


def shard_of(rank: int, world: int, per_rank: int):
    """Global sequence indices owned by `rank` when each rank decodes per_rank sequences."""
    return list(range(rank * per_rank, (rank + 1) * per_rank))


def aggregate(values_per_rank, times_per_rank):
    """Whole-job throughput: all units over the slowest rank's time."""
    t = max(times_per_rank)
    return sum(values_per_rank) / t, t


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


DECODE_SOURCES = ("decode.cu", "decode_tc.cu", "ptx.cuh", "internal.h")
PREFILL_SOURCES = ("prefill.cu", "ptx.cuh", "internal.h")
MLA_SOURCES = ("mla_tc.cu", "ptx.cuh", "internal.h", "mla.h")


def kernel_source_digest(files=DECODE_SOURCES) -> str:
    """Short hash of the sources that define a kernel; ties an ncu summary to the code it measured."""
    h = hashlib.sha256()
    for f in files:
        p = os.path.join(ROOT, "grouped_query_attention_02_b200", "csrc", f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def profile_traffic(name: str, files=DECODE_SOURCES):
    """dram read+write bytes per launch from a committed ncu summary (profiles/<name>), or None
    when the summary is missing or was taken on different kernel sources."""
    import re

    try:
        text = open(os.path.join(PROFILES, name)).read()
    except OSError:
        return None
    dig = re.search(r"kernel_source_digest:\s*([0-9a-f]+)", text)
    val = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not dig or not val or dig.group(1) != kernel_source_digest(files):
        return None
    return int(val.group(1))


class ClockSampler:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- GPU measurement

def _events(torch):
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def time_decode(gqa, torch, x, steps: int, warmup: int, expanded=None):
    """Mean step time and mean split-kernel time (ms) over `steps` timed decode steps."""
    out = torch.empty_like(x.q)
    if hasattr(x, "k_scale"):      # an FP8 cache
        call = lambda: gqa.gqa_decode_fp8(x.q, x.k_cache, x.v_cache, x.seqlens, x.k_scale, x.v_scale, x.scale,
                                          out=out)
    elif expanded is None:
        call = lambda: gqa.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, out=out)
    else:
        call = lambda: gqa.gqa_decode_expanded(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, out=out,
                                               k_rep=expanded[0], v_rep=expanded[1])
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    s0, s1 = _events(torch)
    launches = 0
    s0.record()
    for i in range(steps):
        call()
        launches += gqa.gqa_last_launch_count()
    s1.record()
    torch.cuda.synchronize()
    step_ms = s0.elapsed_time(s1) / steps
    kev = [_events(torch) for _ in range(steps)]
    for i in range(steps):
        gqa.gqa_set_profile_events(*kev[i])
        call()
    gqa.gqa_set_profile_events(None, None)
    torch.cuda.synchronize()
    kern_ms = sum(a.elapsed_time(b) for a, b in kev) / steps
    return step_ms, kern_ms, launches, out


def time_decode_graph(gqa, torch, x, calls: int = 20, replays: int = 50):
    """Mean step time (ms) of the decode replayed from a CUDA graph that captured `calls` calls (the
    serving loop's form: no host work per step)."""
    out = torch.empty_like(x.q)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for _ in range(3):
            decode_call(gqa, x, out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(calls):
            decode_call(gqa, x, out)
    g.replay()
    torch.cuda.synchronize()
    s0, s1 = _events(torch)
    s0.record()
    for _ in range(replays):
        g.replay()
    s1.record()
    torch.cuda.synchronize()
    return s0.elapsed_time(s1) / (replays * calls)


def time_prefill(gqa, torch, p, steps: int, warmup: int):
    out = torch.empty_like(p.q)
    for _ in range(warmup):
        gqa.gqa_prefill_causal(p.q, p.k, p.v, out=out)
    torch.cuda.synchronize()
    kev = [_events(torch) for _ in range(steps)]
    s0, s1 = _events(torch)
    launches = 0
    s0.record()
    for i in range(steps):
        gqa.gqa_set_profile_events(*kev[i])
        gqa.gqa_prefill_causal(p.q, p.k, p.v, out=out)
        launches += gqa.gqa_last_launch_count()
    s1.record()
    gqa.gqa_set_profile_events(None, None)
    torch.cuda.synchronize()
    return s0.elapsed_time(s1) / steps, sum(a.elapsed_time(b) for a, b in kev) / steps, launches


def prefill_backward_flops(B: int, S: int, Hq: int, d: int) -> int:
    """10 * d per unmasked (query, key) pair per head: the five products of the backward
    (S, dP, dV, dK, dQ), the minimal count (recomputation is not counted)."""
    return 10 * d * B * Hq * S * (S + 1) // 2


def time_backward(gqa, torch, inputs, p, steps: int, warmup: int):
    """Mean time (ms) of gqa_prefill_causal_bwd (its three kernels) on the forward's outputs."""
    B, S, Hq, d = p.q.shape
    dout = inputs.make_dout(B, S, Hq, d, device="cuda", seed=0)
    out, lse = gqa.gqa_prefill_causal_fwd(p.q, p.k, p.v)
    dq, dk, dv = torch.empty_like(p.q), torch.empty_like(p.k), torch.empty_like(p.v)
    call = lambda: gqa.gqa_prefill_causal_bwd(p.q, p.k, p.v, out, lse, dout, dq, dk, dv)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    s0, s1 = _events(torch)
    launches = 0
    s0.record()
    for _ in range(steps):
        call()
        launches += gqa.gqa_last_launch_count()
    s1.record()
    torch.cuda.synchronize()
    return s0.elapsed_time(s1) / steps, launches


def mla_decode_flops(B: int, Hq: int, T: int, d_c: int, d_r: int) -> int:
    """2 * Hq * ((d_c + d_r) + d_c) per cached token: every head's score over the whole row and its
    weighted sum of the latent part."""
    return 2 * Hq * (2 * d_c + d_r) * B * T


def time_mla(gqa, torch, x, steps: int, warmup: int):
    """Mean step time and mean decode-kernel time (ms) of gqa_mla_decode."""
    B, Hq, _ = x.q.shape
    out = torch.empty((B, Hq, x.d_c), dtype=torch.bfloat16, device=x.q.device)
    call = lambda: gqa.gqa_mla_decode(x.q, x.kv_cache, x.seqlens, x.scale, out=out, d_c=x.d_c)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    s0, s1 = _events(torch)
    launches = 0
    s0.record()
    for _ in range(steps):
        call()
        launches += gqa.gqa_last_launch_count()
    s1.record()
    torch.cuda.synchronize()
    kev = [_events(torch) for _ in range(steps)]
    for i in range(steps):
        gqa.gqa_set_profile_events(*kev[i])
        call()
    gqa.gqa_set_profile_events(None, None)
    torch.cuda.synchronize()
    return s0.elapsed_time(s1) / steps, sum(a.elapsed_time(b) for a, b in kev) / steps, launches


def decode_call(gqa, x, out, q=None, k=None, v=None, sl=None):
    """One decode step through the public API: the FP8 entry point when x carries per-tensor scales."""
    q = x.q if q is None else q
    k = x.k_cache if k is None else k
    v = x.v_cache if v is None else v
    sl = x.seqlens if sl is None else sl
    if hasattr(x, "k_scale"):
        return gqa.gqa_decode_fp8(q, k, v, sl, x.k_scale, x.v_scale, x.scale, out=out)
    return gqa.gqa_decode(q, k, v, sl, x.scale, out=out)


def time_e2e(gqa, torch, x, steps: int):
    """Host buffers in, host result out: pinned H2D of q, K, V, seqlens + decode + D2H of out, per step."""
    hq = x.q.cpu().pin_memory()
    hk = x.k_cache.cpu().pin_memory()
    hv = x.v_cache.cpu().pin_memory()
    hs = x.seqlens.cpu().pin_memory()
    hout = torch.empty(x.q.shape, dtype=torch.bfloat16).pin_memory()
    dq, dk, dv, ds = (torch.empty_like(t, device="cuda") for t in (hq, hk, hv, hs))
    dout = torch.empty_like(dq)

    def step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        ds.copy_(hs, non_blocking=True)
        decode_call(gqa, x, dout, dq, dk, dv, ds)
        hout.copy_(dout, non_blocking=True)

    step()
    torch.cuda.synchronize()
    s0, s1 = _events(torch)
    s0.record()
    for _ in range(steps):
        step()
    s1.record()
    torch.cuda.synchronize()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hs))
    d2h = hout.numel() * hout.element_size()
    ok = torch.equal(hout, dout.cpu())
    del dq, dk, dv, ds, dout
    return s0.elapsed_time(s1) / steps, h2d, d2h, ok


def cpu_oracle_sample(x, target_s: float = 12.0, gpu_out=None):
    """Time the fp64 oracle on a bounded sample of the workload: the first n sequences (every
    query head), repeated until about target_s seconds of wall time have been spent.  With the GPU's
    output of the same workload (host tensor [B, Hq, d]) the result also carries "parity": the GPU's
    error on the sampled sequences against the oracle's output from the last timed run."""
    import numpy as np
    import oracle

    sl = x.seqlens.cpu().tolist()
    Hkv, d = x.k_cache.shape[2], x.k_cache.shape[3]
    B = len(sl)
    cores = oracle.default_threads()

    def run(n):
        T = max(1, max(sl[:n]))
        q = x.q[:n].cpu()
        kk = x.k_cache[:n, :T].cpu()
        vv = x.v_cache[:n, :T].cpu()
        t0 = time.perf_counter()
        if hasattr(x, "k_scale"):
            r = oracle.decode_fp8(q, kk, vv, x.k_scale, x.v_scale, sl[:n], x.scale, nthreads=cores)
        else:
            r = oracle.decode(q, kk, vv, sl[:n], x.scale, nthreads=cores)
        el = time.perf_counter() - t0
        last["n"], last["ref"] = n, r
        return el

    last = {}

    t1 = run(1)
    n = max(1, min(B, int(target_s / max(t1, 1e-3))))
    reps, spent = 0, 0.0
    while spent < target_s and reps < 1000:
        spent += run(n)
        reps += 1
    ub = unique_kv_bytes(sl[:n], Hkv, d, x.k_cache.element_size()) * reps
    res = {"value": ub / spent / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
           "sample": f"first {n} of {B} sequences (every query head, {sum(sl[:n])} cached tokens) "
                     f"x {reps} repetitions; {spent:.1f} s wall on {cores} threads",
           "seconds": spent, "tokens_per_s": n * reps / spent}
    if gpu_out is not None and "ref" in last:
        ref = last["ref"]
        got = gpu_out[:last["n"]].double().numpy()
        err = np.abs(got - ref)
        rmax = float(np.abs(ref).max())
        res["parity"] = {"max_abs": float(err.max()), "rel_normwise": float(err.max() / rmax) if rmax > 0 else 0.0,
                         "bar": {"max_abs": 2e-2, "rel_normwise": 2e-2},
                         "within_bar": bool(err.max() <= 2e-2 and (rmax == 0 or err.max() / rmax <= 2e-2)),
                         "sample": f"first {last['n']} of {B} sequences, every query head, against the fp64 oracle"}
    return res


def decode_kernel_name(g: int, fp8: bool = False) -> str:
    """Which decode kernel the library launches for group size g (label only): template arguments
    <product width N, FP8 cache, heads per softmax warpgroup, softmax warpgroups>."""
    if fp8 or 3 <= g <= 32:
        n, hw, nwg = (16, 4, 1) if g <= 4 else (16, 8, 1) if g <= 8 else \
            ((16, 8, 2) if fp8 else (16, 16, 1)) if g <= 16 else (32, 16, 2)
        return f"decode_persistent_kernel<{n}, {str(fp8).lower()}, {hw}, {nwg}>"
    return f"decode_split_kernel<{1 if g <= 1 else 2 if g <= 2 else 4 if g <= 4 else 8}>"


def prefill_only(gqa, torch, inputs, workloads, args):
    """Time the causal prefill workload alone (B sequences of 8192 tokens, 32/8 heads, d=128)."""
    pw = workloads.CAUSAL_PREFILL
    peaks = load_peaks()
    hq, hkv = (int(v) for v in args.prefill_heads.split(":"))
    p = inputs.make_prefill(args.prefill_batch, pw.S, hq, hkv, pw.d, device="cuda", seed=0)
    st_ms, k_ms, n = time_prefill(gqa, torch, p, args.steps, args.warmup)
    fl = prefill_causal_flops(args.prefill_batch, pw.S, hq, pw.d)
    print(json.dumps({"metric": "causal GQA prefill TFLOP/s", "value": fl / (st_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": st_ms,
                      "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": pw.name, "B": args.prefill_batch, "Hq": hq, "Hkv": hkv},
                      "roofline": {"bound": "tensor", "achieved": fl / (k_ms * 1e-3) / 1e12,
                                   "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                   "frac": fl / (k_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]},
                      "gpu_launches": n, "device_status": gqa.gqa_get_last_device_status()}))


def mla_roofline(peaks, mw, st_ms, k_ms):
    """The MLA row: tensor-bound at 128 heads (about 242 FLOP per byte, near the ridge), so the target
    time is the larger of FLOP / tensor peak and bytes / HBM peak; both fractions are reported."""
    fl = mla_decode_flops(mw.B, mw.Hq, mw.Tmax, mw.d_c, mw.d_r)
    by = mw.B * mw.Tmax * (mw.d_c + mw.d_r) * 2 + mw.B * mw.Hq * (2 * (mw.d_c + mw.d_r) + 2 * mw.d_c)
    t_bound = max(fl / (peaks["bf16_tflops"] * 1e12), by / (peaks["hbm_gbs"] * 1e9))
    return {
        "ms_per_step": st_ms, "kernel_ms": k_ms, "TFLOPs": fl / (st_ms * 1e-3) / 1e12,
        "unique_kv_GBps": by / (st_ms * 1e-3) / 1e9, "tokens_per_s": mw.B / (st_ms * 1e-3),
        "roofline": {"bound": "tensor", "achieved": fl / (k_ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": fl / (k_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                     "traffic": profile_traffic("mla_decode_deepseek_b32.md", MLA_SOURCES),
                     "hbm_frac": by / (k_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "frac_of_bound": t_bound / (k_ms * 1e-3), "bound_ms": t_bound * 1e3,
                     "peak_source": f"{peaks.get('source')} bf16_tflops (cuBLAS burst), hbm_gbs"},
        "flop_count": "2 Hq (2 d_c + d_r) per cached token; bytes: the cache once, q in, out",
        "kernel": "tcgen05, 64 heads per CTA, persistent, device-planned pieces + combine"}


def mla_only(gqa, torch, inputs, workloads, args):
    """Time the DeepSeek-V3-shaped MLA decode alone (used for its ncu captures)."""
    mw = workloads.MLA_DECODE
    peaks = load_peaks()
    xm = inputs.make_mla_decode(mw.B, mw.Hq, mw.Tmax, mw.d_c, mw.d_r, device="cuda", seed=0)
    st_ms, k_ms, n = time_mla(gqa, torch, xm, args.steps, args.warmup)
    row = mla_roofline(peaks, mw, st_ms, k_ms)
    print(json.dumps({"metric": "MLA absorbed decode TFLOP/s", "value": row["TFLOPs"], "unit": "TFLOP/s",
                      "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": st_ms,
                      "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": mw.name}, "row": row, "gpu_launches": n,
                      "device_status": gqa.gqa_get_last_device_status()}))


def tp_bench(gqa, torch, inputs, args, w, world: int, rank: int, local_rank: int):
    """Tensor-parallel decode of one layer over `world` ranks (one per GPU, NCCL): each rank keeps its head
    shard (a replica of its KV head when Hkv < world), decodes it and all-gathers the outputs in head order.
    Total work is fixed as ranks are added ("strong"); value = the layer's unique KV bytes over the slowest
    rank's step time.  Ranks that hold replicas read the same KV head, so bytes read over all ranks exceed
    the unique bytes; both are reported."""
    import datetime

    import torch.distributed as dist

    from grouped_query_attention_02_b200 import tp as tpmod

    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        # every rank draws the same layer and keeps its shard, as a rank of a deployment holds only its own
        x = inputs.make_decode(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device="cuda", seed=0, seqlen_range=w.seqlen_range)
        shard = tpmod.tp_shard(w.Hq, w.Hkv, world, rank)
        qs, ks, vs = tpmod.take_shard(x.q, x.k_cache, x.v_cache, shard)
        sl, scale = x.seqlens, x.scale
        lens = sl.cpu().tolist()
        del x
        torch.cuda.empty_cache()
        U = unique_kv_bytes(lens, w.Hkv, w.d)
        read_all = unique_kv_bytes(lens, shard.kv_count, w.d) * world
        step = lambda: tpmod.tp_decode(qs, ks, vs, sl, scale, world)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0, s1 = _events(torch)
        with ClockSampler(local_rank) as clk:
            time.sleep(0.25)
            s0.record()
            for _ in range(args.steps):
                out = step()
            s1.record()
            torch.cuda.synchronize()
        ms = s0.elapsed_time(s1) / args.steps
        if world > 1:
            dist.barrier()
            t = torch.tensor([ms], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        ms_max = ms
        if rank == 0:
            print(json.dumps({
                "metric": METRIC + " (tensor-parallel)", "value": U / (ms_max * 1e-3) / 1e9, "unit": "GB/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": {"workload": w.name, "parallelism": f"tp{world} (head shards; KV heads replicated when "
                                                              f"Hkv < tp; outputs all-gathered over NCCL)",
                           "q_heads_per_rank": shard.q_count, "kv_heads_per_rank": shard.kv_count},
                "bytes_read_all_ranks": read_all, "unique_kv_bytes": U,
                "tokens_per_s": w.B / (ms_max * 1e-3), "out_shape": list(out.shape),
                "clocks": clk.summary(), "device_status": gqa.gqa_get_last_device_status()}))
    finally:
        if world > 1:
            dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--rows", choices=["all", "none"], default="all")
    ap.add_argument("--e2e-steps", type=int, default=3, help="0 skips the host-buffer measurement")
    ap.add_argument("--cpu-baseline", choices=["on", "off"], default="on")
    ap.add_argument("--mode", choices=["decode", "prefill", "backward", "mla"], default="decode",
                    help="prefill / backward / mla: time only the causal prefill workload's forward / backward, "
                         "or the MLA decode workload (used for their ncu captures)")
    ap.add_argument("--prefill-batch", type=int, default=4, help="sequences in --mode prefill")
    ap.add_argument("--prefill-heads", default="32:8", help="Hq:Hkv of --mode prefill (e.g. 24:8 for an odd group)")
    ap.add_argument("--decode-workload", default="Qwen3-8B",
                    help="name prefix of the decode workload timed as the headline (profiling other rows)")
    ap.add_argument("--tp", action="store_true",
                    help="tensor-parallel decode of the workload over WORLD_SIZE ranks (head shards, outputs "
                         "all-gathered) instead of the batch-sharded default")
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16",
                    help="fp8: the headline decode over an FP8 (E4M3) cache with per-tensor scales")
    args = ap.parse_args()

    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print(f"--gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    from grouped_query_attention_02_b200 import inputs, workloads

    w = next(x for x in workloads.DECODE_WORKLOADS if x.name.startswith(args.decode_workload))
    fp8 = args.kv == "fp8"
    base_cfg = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.Tmax,
                "global_batch": w.B * max(world, 1), "parallelism": f"dp{max(world, 1)} (batch-sharded, no collective)",
                "kv_cache": "fp8 e4m3, per-tensor scales" if fp8 else "bf16",
                "l2": "inputs larger than L2 (cache of at least 0.8 GB vs 126 MB); no flush"}

    if args.impl == "reference":
        # the reference arm is the fp64 CPU oracle, on rank 0 only
        if rank != 0:
            return
        import oracle

        # inputs on the host: one sequence per step keeps a step to a few seconds
        xs = inputs.make_decode(2, w.Hq, w.Hkv, w.d, w.Tmax, device="cpu", seed=0)
        cores = oracle.default_threads()
        times = []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            oracle.decode(xs.q[:1], xs.k_cache[:1], xs.v_cache[:1], xs.seqlens[:1], xs.scale, nthreads=cores)
            dt = time.perf_counter() - t0
            if i >= args.warmup:
                times.append(dt)
        t = sum(times) / len(times)
        ub = unique_kv_bytes([w.Tmax], w.Hkv, w.d)
        val = ub / t / 1e9
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": base_cfg,
                "cpu_baseline": {"value": val, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                 "sample": f"one of {w.B} sequences per step (all {w.Hq} query heads, "
                                           f"{w.Tmax} cached tokens)"},
                "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import grouped_query_attention_02_b200 as gqa

    gqa.load()
    torch.cuda.set_device(local_rank)
    if args.mode == "prefill":
        prefill_only(gqa, torch, inputs, workloads, args)
        return
    if args.mode == "mla":
        mla_only(gqa, torch, inputs, workloads, args)
        return
    if args.tp:
        tp_bench(gqa, torch, inputs, args, w, max(world, 1), rank, local_rank)
        return
    if args.mode == "backward":
        pw = workloads.CAUSAL_PREFILL
        p = inputs.make_prefill(args.prefill_batch, pw.S, pw.Hq, pw.Hkv, pw.d, device="cuda", seed=0)
        st_ms, n = time_backward(gqa, torch, inputs, p, args.steps, args.warmup)
        fl = prefill_backward_flops(args.prefill_batch, pw.S, pw.Hq, pw.d)
        peaks = load_peaks()
        print(json.dumps({"metric": "causal GQA prefill backward TFLOP/s", "value": fl / (st_ms * 1e-3) / 1e12,
                          "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": st_ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                          "config": {"workload": pw.name, "B": args.prefill_batch},
                          "frac_bf16_peak": fl / (st_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                          "gpu_launches": n, "device_status": gqa.gqa_get_last_device_status()}))
        return
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    peaks = load_peaks()
    make = inputs.make_decode_fp8 if fp8 else inputs.make_decode
    x = make(w.B, w.Hq, w.Hkv, w.d, w.Tmax, device="cuda", seed=rank_seed(rank), seqlen_range=w.seqlen_range)
    sl = x.seqlens.cpu().tolist()
    U = unique_kv_bytes(sl, w.Hkv, w.d, x.k_cache.element_size())
    alg_bytes = U + 2 * x.q.numel() * 2   # cache + q in + out

    # warm-up + barrier, then the timed steps bracketed by barrier + synchronize
    out = torch.empty_like(x.q)
    for _ in range(args.warmup):
        decode_call(gqa, x, out)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    s0, s1 = _events(torch)
    launches = 0
    with ClockSampler(local_rank) as clk:
        time.sleep(0.25)
        s0.record()
        for i in range(args.steps):
            decode_call(gqa, x, out)
            launches += gqa.gqa_last_launch_count()
        s1.record()
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    step_ms = s0.elapsed_time(s1) / args.steps
    # the dominant kernel alone: a second pass with the library's event hook around it (the hook's
    # event records sit between the launches, so this pass is not the step time)
    kev = [_events(torch) for _ in range(args.steps)]
    for i in range(args.steps):
        gqa.gqa_set_profile_events(*kev[i])
        decode_call(gqa, x, out)
    gqa.gqa_set_profile_events(None, None)
    torch.cuda.synchronize()
    kern_ms = sum(a.elapsed_time(b) for a, b in kev) / args.steps
    if dist:
        t = torch.tensor([step_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        step_ms_max = float(t.item())
    else:
        step_ms_max = step_ms
    status = gqa.gqa_get_last_device_status()
    value = U * max(world, 1) / (step_ms_max * 1e-3) / 1e9
    tokens_per_s = w.B * max(world, 1) / (step_ms_max * 1e-3)

    # ---- end to end through the public API with host buffers (every rank; slowest rank counts)
    e2e_err = None
    if args.e2e_steps > 0:
        try:
            e2e_ms, h2d, d2h, ok = time_e2e(gqa, torch, x, args.e2e_steps)
        except RuntimeError as e:  # pinned memory exhausted, etc.
            e2e_ms, h2d, d2h, ok, e2e_err = float("nan"), 0, 0, False, str(e)[:200]
    else:
        e2e_ms, h2d, d2h, ok, e2e_err = float("nan"), 0, 0, False, "skipped (--e2e-steps 0)"
    if dist:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())

    if rank != 0:
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return

    achieved = alg_bytes / (kern_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": max(world, 1), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8 e4m3 cache, f16 products" if fp8 else "bf16", "accumulate": "fp32",
        "data": "synthetic", "config": base_cfg,
        "tokens_per_s": tokens_per_s, "frac_of_hbm_peak_step": value / max(world, 1) / peaks["hbm_gbs"],
        "gpu_launches": launches, "device_status": status,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "traffic": profile_traffic("decode_persistent_fp8_qwen3_8b.md" if fp8 and w is workloads.QWEN3_8B_DECODE
                                                else "decode_persistent_qwen3_8b.md" if w is workloads.QWEN3_8B_DECODE
                                                else "-"),
                     "kernel": decode_kernel_name(w.group, fp8), "kernel_ms": kern_ms, "algorithmic_bytes": alg_bytes,
                     "peak_source": f"{peaks.get('source')} hbm_gbs (copy bandwidth)"},
        "clocks": clk.summary(),
    }

    line["e2e"] = {"value": (U * max(world, 1) / (e2e_ms * 1e-3) / 1e9) if e2e_err is None else None,
                   "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                   "result_matches_device": ok}
    if e2e_err:
        line["e2e"]["error"] = e2e_err

    out_host = out.float().cpu()   # the headline's output, for the parity figure of the CPU-baseline leg

    # ---- the other rows of the hot path
    if args.rows == "all" and max(world, 1) == 1 and not fp8:
        rows = {}
        del out
        for ww in (workloads.TINY_DECODE,) + workloads.VARLEN_DECODE + (workloads.EXTREME_GROUP_DECODE,):
            xx = inputs.make_decode(ww.B, ww.Hq, ww.Hkv, ww.d, ww.Tmax, device="cuda", seed=0,
                                    seqlen_range=ww.seqlen_range)
            sll = xx.seqlens.cpu().tolist()
            uu = unique_kv_bytes(sll, ww.Hkv, ww.d)
            st_ms, k_ms, n, _ = time_decode(gqa, torch, xx, 10 if ww.B * ww.Tmax > 1e5 else 50, 3)
            rows[ww.name] = {"ms_per_step": st_ms, "kernel_ms": k_ms, "unique_kv_GBps": uu / (st_ms * 1e-3) / 1e9,
                             "kernel_frac_hbm": uu / (k_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                             "frac_hbm": uu / (st_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                             "tokens_per_s": ww.B / (st_ms * 1e-3), "launches_per_step": n / (10 if ww.B * ww.Tmax > 1e5 else 50)}
            if ww is workloads.TINY_DECODE:
                rows[ww.name]["graph_ms_per_step"] = time_decode_graph(gqa, torch, xx)
            del xx
            torch.cuda.empty_cache()
        # expanded repeat-KV baseline on the headline workload
        k_rep = torch.empty((w.B, w.Tmax, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
        v_rep = torch.empty_like(k_rep)
        st_ms, k_ms, n, _ = time_decode(gqa, torch, x, 5, 2, expanded=(k_rep, v_rep))
        rows["expanded repeat-KV baseline, " + w.name] = {
            "ms_per_step": st_ms, "unique_kv_GBps": U / (st_ms * 1e-3) / 1e9,
            "bytes_moved_per_step": U + 2 * U * w.group + U * w.group,
            "slowdown_vs_grouped": st_ms / step_ms}
        del k_rep, v_rep
        torch.cuda.empty_cache()
        # FP8 (E4M3) caches: half the bytes per token
        for ww in (w, workloads.VARLEN_DECODE[1], workloads.VARLEN_DECODE[3], workloads.EXTREME_GROUP_DECODE):
            xx = inputs.make_decode_fp8(ww.B, ww.Hq, ww.Hkv, ww.d, ww.Tmax, device="cuda", seed=0,
                                        seqlen_range=ww.seqlen_range)
            uu = unique_kv_bytes(xx.seqlens.cpu().tolist(), ww.Hkv, ww.d, elem_bytes=1)
            st_ms, k_ms, n, _ = time_decode(gqa, torch, xx, 20, 3)
            rows["FP8 KV cache, " + ww.name] = {
                "ms_per_step": st_ms, "kernel_ms": k_ms, "unique_kv_GBps": uu / (st_ms * 1e-3) / 1e9,
                "kernel_frac_hbm": uu / (k_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "frac_hbm": uu / (st_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "tokens_per_s": ww.B / (st_ms * 1e-3), "launches_per_step": n / 20,
                "speedup_vs_bf16_cache": (rows.get(ww.name, {}).get("ms_per_step") or
                                          (step_ms if ww is w else float("nan"))) / st_ms}
            del xx
            torch.cuda.empty_cache()
        # causal prefill
        pw = workloads.CAUSAL_PREFILL
        try:
            p = inputs.make_prefill(pw.B, pw.S, pw.Hq, pw.Hkv, pw.d, device="cuda", seed=0)
            st_ms, k_ms, n = time_prefill(gqa, torch, p, 10, 3)
            fl = prefill_causal_flops(pw.B, pw.S, pw.Hq, pw.d)
            t1 = profile_traffic("prefill_causal_b1_s8192.md", PREFILL_SOURCES)
            rows[pw.name] = {"ms_per_step": st_ms, "kernel_ms": k_ms, "TFLOPs": fl / (st_ms * 1e-3) / 1e12,
                             "roofline": {"bound": "tensor", "achieved": fl / (k_ms * 1e-3) / 1e12,
                                          "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                          "frac": fl / (k_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                          "traffic": None if t1 is None else t1 * pw.B,
                                          "traffic_note": "ncu capture at B=1 scaled by B (traffic is per sequence)",
                                          "peak_source": f"{peaks.get('source')} bf16_tflops (cuBLAS burst)"}}
        except gqa.GQAError as e:
            rows[pw.name] = {"error": str(e)}
        # the same prefill with an odd group (24 query / 8 KV heads, g = 3): query tiles 2k, 2k+1 of one head per CTA
        try:
            name = "causal GQA prefill, odd group B4 S8192 Hq24 Hkv8 d128"
            p = inputs.make_prefill(pw.B, pw.S, 24, 8, pw.d, device="cuda", seed=0)
            st_ms, k_ms, n = time_prefill(gqa, torch, p, 10, 3)
            fl = prefill_causal_flops(pw.B, pw.S, 24, pw.d)
            rows[name] = {"ms_per_step": st_ms, "kernel_ms": k_ms, "TFLOPs": fl / (st_ms * 1e-3) / 1e12,
                          "kernel": "prefill_pair_kernel, query-tile pairs (odd group)",
                          "roofline": {"bound": "tensor", "achieved": fl / (k_ms * 1e-3) / 1e12,
                                       "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                       "frac": fl / (k_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], "traffic": None,
                                       "peak_source": f"{peaks.get('source')} bf16_tflops (cuBLAS burst)"}}
            del p
            torch.cuda.empty_cache()
        except gqa.GQAError as e:
            rows["causal GQA prefill, odd group"] = {"error": str(e)}
        # causal prefill backward (dq, and dk / dv summed over each group)
        try:
            p = inputs.make_prefill(pw.B, pw.S, pw.Hq, pw.Hkv, pw.d, device="cuda", seed=0)
            st_ms, n = time_backward(gqa, torch, inputs, p, 5, 2)
            fl = prefill_backward_flops(pw.B, pw.S, pw.Hq, pw.d)
            rows["backward, " + pw.name] = {
                "ms_per_step": st_ms, "TFLOPs": fl / (st_ms * 1e-3) / 1e12,
                "frac_bf16_peak": fl / (st_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                "flop_count": "10 d per unmasked pair per head (five products; recomputed S, dP not counted)",
                "launches_per_step": n / 5}
            del p
            torch.cuda.empty_cache()
        except gqa.GQAError as e:
            rows["backward, " + pw.name] = {"error": str(e)}
        # MLA decode with absorbed weights (tensor cores)
        mw = workloads.MLA_DECODE
        try:
            xm = inputs.make_mla_decode(mw.B, mw.Hq, mw.Tmax, mw.d_c, mw.d_r, device="cuda", seed=0)
            st_ms, k_ms, n = time_mla(gqa, torch, xm, 20, 3)
            rows[mw.name] = mla_roofline(peaks, mw, st_ms, k_ms)
            rows[mw.name]["launches_per_step"] = n / 20
            del xm
            torch.cuda.empty_cache()
        except (gqa.GQAError, RuntimeError) as e:   # a row that fails must not cost the line
            rows[mw.name] = {"error": f"{type(e).__name__}: {e}"}
        line["rows"] = rows

    # ---- the fp64 oracle on a bounded sample, host cores of this machine
    if max(world, 1) == 1 and args.cpu_baseline == "on":
        cb = cpu_oracle_sample(x, gpu_out=out_host)
        parity = cb.pop("parity", None)
        line["cpu_baseline"] = cb
        if parity is not None:
            line["parity"] = parity

    print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
