"""Benchmark of the MiMo-V2-Flash hybrid attention hot path on B200.

One step = one pass over every kernel of the path at the model's head shape
(64 query heads, 4 key/value heads, head dims 192 / 128), seeded synthetic
bf16 inputs ~N(0, 1), fp32 sink logits ~N(0, 1):

  1. sliding-window prefill, T = 32768, window 129      (HBM-bound)
  2. global prefill, T = 32768, causal                   (tensor-core-bound)
  3. global decode, batch 64, lengths ~U[1024, 262144] in 262144-slot caches
     (split-KV + combine; HBM-bound)
  4. sliding-window decode, batch 64, 129-slot ring caches (latency-bound)

Reported value: the step's roofline floor (sum over the four kernels of
max(useful FLOP / bf16 tensor peak, algorithmic bytes / HBM peak), peaks from
MEASURED_PEAKS.json) divided by the measured step time, in % -- summed over
GPUs for N > 1 (each GPU runs its own step: weak scaling, no collective on the
data path).  Per-kernel TFLOP/s and GB/s are in "parts".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "prefill attn TFLOP/s & decode KV-cache GB/s, % of B200 roofline"
UNIT = "% of B200 roofline (sum over GPUs)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

T_PREFILL = 32768
SWA = W.SWA_WINDOW
HQ, HKV, DQK, DV = W.HQ, W.HKV, W.DQK, W.DV
FLOP_PER_PAIR = 2 * DQK + 2 * DV          # per (visible pair, query head)
KV_BYTES_PER_TOKEN = HKV * (DQK + DV) * 2   # 2560 B of K and V per cached token


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- work model

def visible_pairs(T, window):
    if window == 0:
        return T * (T + 1) // 2
    w = window
    return sum(min(i + 1, w) for i in range(T)) if T < 4096 else (
        w * (w + 1) // 2 + (T - w) * w if T >= w else T * (T + 1) // 2)


def prefill_work(T, window):
    flops = FLOP_PER_PAIR * HQ * visible_pairs(T, window)
    byts = T * (HQ * DQK * 2 + HKV * (DQK + DV) * 2 + HQ * DV * 2 + HQ * 4)
    return flops, byts


def varlen_prefill_work(lengths, window, out_bytes=2):
    """prefill_work summed over a packed batch of sequences (one layer)."""
    flops = sum(FLOP_PER_PAIR * HQ * visible_pairs(int(L), window) for L in lengths)
    byts = int(sum(lengths)) * (HQ * DQK * 2 + HKV * (DQK + DV) * 2 + HQ * DV * out_bytes + HQ * 4)
    return flops, byts


def decode_work(lengths, window, capacity):
    ring = window > 0 and capacity == window
    vis = [min(L, capacity) if ring else (min(L, window) if window > 0 else L) for L in lengths]
    flops = FLOP_PER_PAIR * HQ * sum(vis)
    byts = sum(vis) * KV_BYTES_PER_TOKEN + len(lengths) * HQ * (DQK * 2 + DV * 2 + 4)
    return flops, byts


def decode_fp8_work(lengths, window, capacity):
    """decode_work with one byte per cache element (e4m3) plus the 2 x Hkv fp32 scales."""
    flops, byts = decode_work(lengths, window, capacity)
    ring = window > 0 and capacity == window
    vis = [min(L, capacity) if ring else (min(L, window) if window > 0 else L) for L in lengths]
    return flops, byts - sum(vis) * KV_BYTES_PER_TOKEN // 2 + 2 * HKV * 4


def graph_us(fn, n=20, reps=10):
    """Device time per call of a small launch: n calls captured in a CUDA graph and
    replayed (a host call through the Python binding costs ~15-20 us on its own)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / n)
    del g
    return 1e3 * float(np.median(ts[2:]))


class L2Flush:
    """Evicts the 126 MB L2 between timed launches: writes a 256 MB buffer, then
    reads another, so the written (dirty) lines are written back to HBM during
    the read, before the next timed event, and L2 is left holding clean lines."""

    def __init__(self, dev):
        self.w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.max()


def floor_s(flops, byts, peaks):
    return max(flops / (peaks["bf16_tflops"] * 1e12), byts / (peaks["hbm_gbs"] * 1e9))


# ---------------------------------------------------------------- ranks

def max_over_ranks(x, world, device=None):
    """MAX of a per-rank scalar over all ranks (NCCL on GPUs, gloo on CPU)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def step_value(floor_step_ms, max_ms, world):
    """Whole-job value: every rank ran one step (weak scaling), timed as the max over ranks."""
    return 100.0 * world * floor_step_ms / max_ms


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(1.0)  # let nvidia-smi start sampling before the timed region
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        rows = []
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), max=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        load = [r for r in rows if r["power"] > 300] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, peaks, peak_kind):
    import global_attention_swa_b200 as mimo

    dev = torch.device("cuda", torch.cuda.current_device())
    seed = 1000 * rank
    # --- inputs resident in HBM
    swa = W.prefill_inputs([T_PREFILL], seed=seed + 1, device=dev)
    ga = W.prefill_inputs([T_PREFILL], seed=seed + 2, device=dev)
    lengths = W.decode_b64_lengths(0)
    dga = W.decode_inputs(lengths, W.DECODE_GA_CAPACITY, 0, seed=seed + 3, device=dev)
    dsw = W.decode_inputs(lengths, SWA, SWA, seed=seed + 4, device=dev)
    o_swa = torch.empty((T_PREFILL, HQ, DV), dtype=torch.bfloat16, device=dev)
    o_ga = torch.empty_like(o_swa)
    l_swa = torch.empty((HQ, T_PREFILL), dtype=torch.float32, device=dev)
    l_ga = torch.empty_like(l_swa)
    o_dga = torch.empty((64, HQ, DV), dtype=torch.bfloat16, device=dev)
    o_dsw = torch.empty_like(o_dga)
    l_dga = torch.empty((64, HQ), dtype=torch.float32, device=dev)
    l_dsw = torch.empty_like(l_dga)
    ws_ga = torch.empty(max(1, mimo.mimo_attn_decode_workspace_size(
        HQ, HKV, 64, W.DECODE_GA_CAPACITY, 0)), dtype=torch.uint8, device=dev)
    ws_sw = torch.empty(max(1, mimo.mimo_attn_decode_workspace_size(HQ, HKV, 64, SWA, SWA)),
                        dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def step(evs=None):
        rec = (lambda i: evs[i].record(stream)) if evs else (lambda i: None)
        rec(0)
        mimo.mimo_attn_prefill(swa.q, swa.k, swa.v, swa.sinks, SWA, swa.cu_seqlens, T_PREFILL,
                               out=o_swa, lse=l_swa)
        rec(1)
        mimo.mimo_attn_prefill(ga.q, ga.k, ga.v, ga.sinks, 0, ga.cu_seqlens, T_PREFILL,
                               out=o_ga, lse=l_ga)
        rec(2)
        mimo.mimo_attn_decode(dga.q, dga.k_cache, dga.v_cache, dga.seqlens, 0, dga.sinks,
                              out=o_dga, lse=l_dga, workspace=ws_ga)
        rec(3)
        mimo.mimo_attn_decode(dsw.q, dsw.k_cache, dsw.v_cache, dsw.seqlens, SWA, dsw.sinks,
                              out=o_dsw, lse=l_dsw, workspace=ws_sw)
        rec(4)

    launches_per_step = 2 + (2 if ws_ga.numel() > 1 else 1) + (2 if ws_sw.numel() > 1 else 1)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    mimo.mimo_attn_device_status()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t_wall = time.perf_counter()
        for k in range(args.steps):
            flush()                # L2 flush between steps (outside the events)
            step(evs[k])
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if world > 1:
        torch.distributed.barrier()
    mimo.mimo_attn_device_status()

    per = np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(4)]
                    for k in range(args.steps)])  # ms [K, 4]
    step_ms = per.sum(axis=1)
    mean_ms = float(step_ms.mean())
    max_ms = max_over_ranks(mean_ms, world, dev)

    works = [prefill_work(T_PREFILL, SWA), prefill_work(T_PREFILL, 0),
             decode_work(lengths, 0, W.DECODE_GA_CAPACITY), decode_work(lengths, SWA, SWA)]
    floors = [floor_s(f, b, peaks) for f, b in works]
    floor_step_ms = 1e3 * sum(floors)
    value = step_value(floor_step_ms, max_ms, world)
    names = ["prefill_swa_T32768_W129", "prefill_global_T32768", "decode_global_B64_cap262144",
             "decode_swa_ring_B64_W129"]
    bounds = ["hbm", "tensor", "hbm", "hbm"]
    parts = {}
    for i, n in enumerate(names):
        ms = float(per[:, i].mean())
        f, b = works[i]
        parts[n] = {"ms": round(ms, 4), "TFLOP/s": round(f / (ms * 1e-3) / 1e12, 2),
                    "GB/s": round(b / (ms * 1e-3) / 1e9, 1),
                    "roofline_frac": round(1e3 * floors[i] / ms, 4), "bound": bounds[i],
                    "useful_flop": f, "algorithmic_bytes": b}

    # dominant kernel: global prefill (tensor-bound)
    ga_ms = float(per[:, 1].mean())
    ga_tflops = works[1][0] / (ga_ms * 1e-3) / 1e12
    roofline = {"kernel": "prefill_kernel (global, T=32768)", "bound": "tensor",
                "achieved": round(ga_tflops, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(ga_tflops / peaks["bf16_tflops"], 4),
                "peak_kind": f"{peak_kind} burst bf16",
                "frac_of_sustained": round(ga_tflops / peaks["bf16_tflops_sustained"], 4),
                "traffic": None}
    tr = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tr):
        import hashlib

        rec = json.load(open(tr))
        h = hashlib.sha256()
        for f in rec.get("source_files", []):
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
        # counters taken on another revision of the kernel do not describe this one
        if h.hexdigest() == rec.get("source_sha256"):
            roofline["traffic"] = rec.get("prefill_global_T32768")

    # --- e2e through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, mimo, swa, ga, dga, dsw, lengths, dev, floor_step_ms, world,
                      o_swa, o_ga, o_dga, o_dsw, l_swa, l_ga, l_dga, l_dsw, ws_ga, ws_sw)

    # --- the next row outside the step: global decode over e4m3 caches (same
    # lengths and capacity), timed alone after the step's region
    extra = None
    if not args.no_extra:
        del dga
        torch.cuda.empty_cache()
        d8 = W.decode_inputs_fp8(lengths, W.DECODE_GA_CAPACITY, 0, seed=seed + 3, device=dev)
        o8 = torch.empty_like(o_dga)
        l8 = torch.empty_like(l_dga)
        fn = lambda: mimo.mimo_attn_decode_fp8(d8.q, d8.k_codes, d8.v_codes, d8.k_scale,  # noqa: E731
                                               d8.v_scale_kv, d8.seqlens, 0, d8.sinks, out=o8,
                                               lse=l8, workspace=ws_ga)
        ms8 = []
        for i in range(args.warmup + 10):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                ms8.append(e0.elapsed_time(e1))
        mimo.mimo_attn_device_status()
        f8, b8 = decode_fp8_work(lengths, 0, W.DECODE_GA_CAPACITY)
        m8 = float(np.mean(ms8))
        extra = {"decode_global_fp8_B64_cap262144": {
            "ms": round(m8, 4), "GB/s": round(b8 / (m8 * 1e-3) / 1e9, 1),
            "roofline_frac": round(1e3 * floor_s(f8, b8, peaks) / m8, 4), "bound": "hbm",
            "algorithmic_bytes": b8, "launches": 2,
            "note": "e4m3 K/V caches with per-KV-head scales (the next row after the step's "
                    "kernels); not part of the step or its value"}}
        del d8
        # decode-step rotation + append of B=64 new tokens into the 129-slot rings
        # (latency-bound: 3.5 MB moved)
        gq = torch.Generator(device=dev)
        gq.manual_seed(seed + 11)
        qn = torch.randn((64, HQ, DQK), generator=gq, device=dev).to(torch.bfloat16)
        kn = torch.randn((64, HKV, DQK), generator=gq, device=dev).to(torch.bfloat16)
        vn = torch.randn((64, HKV, DV), generator=gq, device=dev).to(torch.bfloat16)
        ra = lambda: mimo.mimo_attn_rope_append(qn, kn, vn, dsw.k_cache, dsw.v_cache,  # noqa: E731
                                                dsw.seqlens, SWA, 10000.0)
        ms_ra = []
        for i in range(args.warmup + 20):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ra()
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                ms_ra.append(e0.elapsed_time(e1))
        us_ra = graph_us(ra)
        mimo.mimo_attn_device_status()
        bytes_ra = 64 * (2 * HQ * DQK * 2 + 2 * HKV * (DQK + DV) * 2)
        extra["rope_append_B64"] = {
            "us": round(us_ra, 2), "GB/s": round(bytes_ra / (us_ra * 1e-6) / 1e9, 1),
            "us_single_host_call": round(1e3 * float(np.median(ms_ra)), 2),
            "algorithmic_bytes": bytes_ra, "launches": 1,
            "note": "rotation of the new token's q (in place) and k, append of k and v to the "
                    "129-slot rings; us = device time per call (CUDA graph replay of 20 calls); "
                    "launch/latency-bound, L2-resident"}

    # context-parallel merge of 8 parts (the gathered per-rank results of a
    # B=64 global decode split over 8 GPUs): one launch, ~2.2 MB read
    if extra is not None:
        gm = torch.Generator(device=dev)
        gm.manual_seed(seed + 13)
        po = torch.randn((8, 64, HQ, DV), generator=gm, device=dev)
        pl = torch.randn((8, 64, HQ), generator=gm, device=dev)
        mo = torch.empty((64, HQ, DV), dtype=torch.bfloat16, device=dev)
        ml = torch.empty((64, HQ), dtype=torch.float32, device=dev)
        us_m = graph_us(lambda: mimo.mimo_attn_decode_merge(po, pl, dsw.sinks, out=mo, lse=ml))
        mimo.mimo_attn_device_status()
        bytes_m = po.numel() * 4 + pl.numel() * 4 + mo.numel() * 2 + ml.numel() * 4
        extra["decode_merge_R8_B64"] = {
            "us": round(us_m, 2), "GB/s": round(bytes_m / (us_m * 1e-6) / 1e9, 1),
            "algorithmic_bytes": bytes_m, "launches": 1,
            "note": "log-sum-exp merge of 8 context-parallel parts with the sink; us = device "
                    "time per call (CUDA graph replay); the all-gather before it is NCCL (not run "
                    "on one GPU)"}

    # prefill backward of one global layer at T=8192 (training; row next-3)
    if extra is not None:
        Tb = 8192
        xb = W.prefill_inputs([Tb], seed=seed + 17, device=dev)
        ob, lb = mimo.mimo_attn_prefill(xb.q, xb.k, xb.v, xb.sinks, 0, xb.cu_seqlens, Tb)
        gb = torch.Generator(device=dev)
        gb.manual_seed(seed + 19)
        dob = torch.randn(ob.shape, generator=gb, device=dev).to(ob.dtype)
        ms_b = []
        for i in range(args.warmup + 5):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            mimo.mimo_attn_prefill_backward(xb.q, xb.k, xb.v, ob, lb, dob, xb.sinks, 0,
                                            xb.cu_seqlens, Tb)
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                ms_b.append(e0.elapsed_time(e1))
        mimo.mimo_attn_device_status()
        pairs = Tb * (Tb + 1) // 2
        fb = 1664 * HQ * pairs  # S, dP, dV, dK, dQ: 2 x (192 + 128 + 128 + 192 + 192) per pair and head
        m_b = float(np.mean(ms_b))
        extra["prefill_backward_global_T8192"] = {
            "ms": round(m_b, 3), "TFLOP/s": round(fb / (m_b * 1e-3) / 1e12, 1),
            "roofline_frac": round(fb / (m_b * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
            "bound": "tensor", "useful_flop": fb, "launches": 4,
            "note": "dq, dk, dv, dsinks (the forward's out and lse as inputs): dQ in one tcgen05 "
                    "pass over 128-key tiles, dK and dV in another (each recomputes S and dP), D "
                    "and the sink gradient in two small launches"}
        del xb, ob, lb, dob

    # varlen 5:1 stack: 16 packed sequences, lengths ~U[512, 8192], six layers
    # (windows 129 x 5, then global) with their own q/k/v and per-layer sinks
    if extra is not None:
        lengths5 = W.varlen_stack_lengths(0)
        nt5, max5 = int(sum(lengths5)), int(max(lengths5))
        sinks5 = W.stack_sinks(len(W.STACK_WINDOWS), seed=seed, device=dev)
        layers = [W.prefill_inputs(lengths5, seed=seed + 30 + i, sinks=False, device=dev)
                  for i in range(len(W.STACK_WINDOWS))]
        outs5 = [torch.empty((nt5, HQ, DV), dtype=torch.bfloat16, device=dev) for _ in layers]
        lses5 = [torch.empty((HQ, nt5), dtype=torch.float32, device=dev) for _ in layers]
        nl = len(layers)
        ms5 = []
        for i in range(args.warmup + 5):
            flush()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)]
            ev[0].record(stream)
            for li, (x, w) in enumerate(zip(layers, W.STACK_WINDOWS)):
                mimo.mimo_attn_prefill(x.q, x.k, x.v, sinks5[li], w, x.cu_seqlens, max5,
                                       out=outs5[li], lse=lses5[li])
                ev[li + 1].record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                ms5.append([ev[j].elapsed_time(ev[j + 1]) for j in range(nl)])
        mimo.mimo_attn_device_status()
        ms5 = np.array(ms5).mean(axis=0)
        w5 = [varlen_prefill_work(lengths5, w) for w in W.STACK_WINDOWS]
        f5 = [floor_s(f, b, peaks) for f, b in w5]
        extra["prefill_varlen_stack_5to1_16seq"] = {
            "ms": round(float(ms5.sum()), 4), "floor_ms": round(1e3 * sum(f5), 4),
            "roofline_frac": round(1e3 * sum(f5) / float(ms5.sum()), 4),
            "layers": [{"window": w, "ms": round(float(m), 4),
                        "TFLOP/s": round(f / (m * 1e-3) / 1e12, 1),
                        "GB/s": round(b / (m * 1e-3) / 1e9, 1),
                        "roofline_frac": round(1e3 * fl / m, 4)}
                       for w, m, (f, b), fl in zip(W.STACK_WINDOWS, ms5, w5, f5)],
            "total_tokens": nt5, "useful_flop": int(sum(f for f, _ in w5)),
            "algorithmic_bytes": int(sum(b for _, b in w5)), "launches": nl,
            "note": "16 sequences, lengths default_rng(0).integers(512, 8193, 16), packed via "
                    "cu_seqlens; layers 0-4 window 129, layer 5 global; bf16 out + lse; L2 "
                    "flushed before each stack pass; floor = sum over layers of max(FLOP / "
                    "tensor peak, bytes / HBM peak)"}
        del layers, outs5, lses5
        # the tiny sliding-window config (T=512, 16/1 heads, fp32 out): launch-bound
        xt = W.prefill_inputs([512], hq=16, hkv=1, seed=seed + 40, device=dev)
        ot = torch.empty((512, 16, DV), dtype=torch.float32, device=dev)
        lt = torch.empty((16, 512), dtype=torch.float32, device=dev)
        us_t = graph_us(lambda: mimo.mimo_attn_prefill(xt.q, xt.k, xt.v, xt.sinks, SWA,
                                                       xt.cu_seqlens, 512, out=ot, lse=lt))
        mimo.mimo_attn_device_status()
        extra["prefill_tiny_swa_T512_H16"] = {
            "us": round(us_t, 2), "launches": 1,
            "note": "T=512, 16 query heads over 1 key/value head, window 129, fp32 out; device "
                    "time per call (CUDA graph replay of 20 calls); launch/latency-bound"}

    res = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v, N(0,1) fp32 sinks)",
        "config": {"workload": "hybrid attention step at model head shape: SWA prefill "
                               "T=32768 W=129 + global prefill T=32768 + decode B=64 (global, "
                               "262144-slot caches, lengths ~U[1024,262144]) + decode B=64 "
                               "(129-slot SWA ring)",
                   "heads_q": HQ, "heads_kv": HKV, "head_dim_qk": DQK, "head_dim_v": DV,
                   "seq_len": T_PREFILL, "decode_batch": 64, "parallelism": f"replicas{world}",
                   "l2": "flushed between steps (256 MB write, then a 256 MB read that "
                         "writes the dirty lines back before the first event); every input > L2 "
                         "except the "
                         "21 MB ring caches",
                   "floor_ms_per_step": round(floor_step_ms, 4),
                   "peaks": {**peaks, "source": peak_kind}},
        "parts": parts,
        "extra": extra,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "wall_s_timed_region": round(t_wall, 4),
    }
    return res


def run_e2e(args, mimo, swa, ga, dga, dsw, lengths, dev, floor_step_ms, world,
            o_swa, o_ga, o_dga, o_dsw, l_swa, l_ga, l_dga, l_dsw, ws_ga, ws_sw):
    """Same step through the public API, inputs copied from pinned host memory each
    step and every output read back.  KV caches are the decode layers' persistent
    state and stay resident; the decode step's input is the new query.

    Copies overlap compute: host->device copies run on their own stream into one of
    two device input sets (the next step's inputs load while this step computes),
    device->host reads of each kernel's outputs run on a third stream as soon as
    that kernel is done, into one of two device output sets.  The host link's
    host->device direction bounds the step (1.78 GB of inputs), so a step loads
    the decode queries first, then the global layer's q/k/v, then the sliding-
    window layer's: the long global prefill starts half-way through the step's
    copies and overlaps the rest, and only the short sliding-window prefill and
    the two output reads are left after the last input lands."""
    names = ("sq", "sk", "sv", "gq", "gk", "gv", "dq", "rq")
    srcs = (swa.q, swa.k, swa.v, ga.q, ga.k, ga.v, dga.q, dsw.q)
    host = {}
    for name, t in zip(names, srcs):
        host[name] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        host[name].copy_(t)
    dev_in = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
    outs_dev = [dict(o_swa=o_swa, l_swa=l_swa, o_ga=o_ga, l_ga=l_ga, o_dga=o_dga, l_dga=l_dga,
                     o_dsw=o_dsw, l_dsw=l_dsw)]
    outs_dev.append({k: torch.empty_like(v) for k, v in outs_dev[0].items()})
    outs_host = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                 for k, v in outs_dev[0].items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_host.values())
    s_h2d, s_cmp, s_d2h = torch.cuda.Stream(), torch.cuda.current_stream(), torch.cuda.Stream()
    ws_reads = [torch.cuda.Event() for _ in range(2)]   # outputs set b read back -> reusable
    in_used = [torch.cuda.Event() for _ in range(2)]    # inputs set b consumed -> reusable

    def step(k):
        b = k & 1
        din, dout = dev_in[b], outs_dev[b]
        loaded = {}
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_event(in_used[b])
            for grp in (("dq", "rq"), ("gq", "gk", "gv"), ("sq", "sk", "sv")):
                for nme in grp:
                    din[nme].copy_(host[nme], non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_h2d)
                loaded[grp[0]] = e
        s_cmp.wait_event(ws_reads[b])
        done = {}
        s_cmp.wait_event(loaded["dq"])
        mimo.mimo_attn_decode(din["dq"], dga.k_cache, dga.v_cache, dga.seqlens, 0, dga.sinks,
                              out=dout["o_dga"], lse=dout["l_dga"], workspace=ws_ga, stream=s_cmp)
        mimo.mimo_attn_decode(din["rq"], dsw.k_cache, dsw.v_cache, dsw.seqlens, SWA, dsw.sinks,
                              out=dout["o_dsw"], lse=dout["l_dsw"], workspace=ws_sw, stream=s_cmp)
        done["dec"] = torch.cuda.Event(); done["dec"].record(s_cmp)
        s_cmp.wait_event(loaded["gq"])
        mimo.mimo_attn_prefill(din["gq"], din["gk"], din["gv"], ga.sinks, 0, ga.cu_seqlens,
                               T_PREFILL, out=dout["o_ga"], lse=dout["l_ga"], stream=s_cmp)
        done["ga"] = torch.cuda.Event(); done["ga"].record(s_cmp)
        s_cmp.wait_event(loaded["sq"])
        mimo.mimo_attn_prefill(din["sq"], din["sk"], din["sv"], swa.sinks, SWA, swa.cu_seqlens,
                               T_PREFILL, out=dout["o_swa"], lse=dout["l_swa"], stream=s_cmp)
        done["swa"] = torch.cuda.Event(); done["swa"].record(s_cmp)
        in_used[b].record(s_cmp)
        with torch.cuda.stream(s_d2h):
            for ev, keys in ((done["dec"], ("o_dga", "l_dga", "o_dsw", "l_dsw")),
                             (done["ga"], ("o_ga", "l_ga")), (done["swa"], ("o_swa", "l_swa"))):
                s_d2h.wait_event(ev)
                for kk in keys:
                    outs_host[kk].copy_(dout[kk], non_blocking=True)
            ws_reads[b].record(s_d2h)

    for k in range(2):
        step(k)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    # every timed step of the kernel leg (at most 30): the last step's tail (its
    # sliding-window prefill and output reads) is spread over all of them
    n = max(2, min(args.steps, 30))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(s_h2d)
    for k in range(n):
        step(k)
    s_h2d.wait_stream(s_d2h)
    s_h2d.wait_stream(s_cmp)
    t1.record(s_h2d)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / n, world, dev)
    return {"value": round(step_value(floor_step_ms, ms, world), 3), "unit": UNIT,
            "ms_per_step": round(ms, 3), "steps": n,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "overlap": "h2d / compute / d2h on three streams, double-buffered device buffers"}


# ---------------------------------------------------------------- oracle arms

class OracleSample:
    """The fp64 oracle on a bounded sample of one step (inputs generated once)."""

    def __init__(self, rows_swa, rows_ga, decode_seqs):
        self.rows_swa, self.rows_ga, self.decode_seqs = rows_swa, rows_ga, decode_seqs
        self.pre = {SWA: W.prefill_inputs([T_PREFILL], seed=1), 0: W.prefill_inputs([T_PREFILL], seed=2)}
        lengths = W.decode_b64_lengths(0)
        self.Ls = [lengths[b] for b in range(decode_seqs)]
        self.dec = [(0, None, W.decode_inputs(self.Ls, max(self.Ls), 0, seed=3, poison=False)),
                    (SWA, SWA, W.decode_inputs(self.Ls, SWA, SWA, seed=4, poison=False))]
        self.sample = (
            f"{rows_swa} random query rows x 64 heads of the T=32768 SWA prefill, {rows_ga} of "
            f"the global prefill, {decode_seqs} of the 64 global-decode sequences and "
            f"{decode_seqs} ring-decode sequence(s); value = roofline floor of the sampled "
            f"work / oracle seconds")

    def run(self, peaks, seed=0):
        import oracle

        t_total = 0.0
        floor_sample = 0.0
        # prefills: random query rows (all 64 heads); the sampled share of pairs / bytes
        for window, nrows in ((SWA, self.rows_swa), (0, self.rows_ga)):
            x = self.pre[window]
            rows = np.sort(np.random.default_rng(seed * 7 + window).choice(
                T_PREFILL, nrows, replace=False))
            t0 = time.perf_counter()
            oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, rows=rows)
            t_total += time.perf_counter() - t0
            pairs = sum(min(int(r) + 1, window) if window else int(r) + 1 for r in rows)
            f = FLOP_PER_PAIR * HQ * pairs
            b = prefill_work(T_PREFILL, window)[1] * nrows / T_PREFILL
            floor_sample += floor_s(f, b, peaks)
        for window, cap, d in self.dec:
            c = d.capacity
            t0 = time.perf_counter()
            oracle.decode(d.q, d.k_cache, d.v_cache, d.seqlens, window, d.sinks,
                          ring=(cap is not None))
            t_total += time.perf_counter() - t0
            f, b = decode_work(self.Ls, window, c)
            floor_sample += floor_s(f, b, peaks)
        return 100.0 * floor_sample / t_total, t_total


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, peaks, peak_kind):
    vals, secs = [], []
    smp = OracleSample(rows_swa=64, rows_ga=8, decode_seqs=1)
    sample = smp.sample
    for i in range(args.warmup + args.steps):
        v, s = smp.run(peaks, seed=i)
        if i >= args.warmup:
            vals.append(v)
            secs.append(s)
    v = float(np.mean(vals))
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * float(np.mean(secs)), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v, N(0,1) fp32 sinks)",
        "config": {"workload": "hybrid attention step at model head shape (bounded sample per "
                               "step, see cpu_baseline.sample)", "peaks": {**peaks, "source": peak_kind}},
        "cpu_baseline": {"value": round(v, 6), "unit": UNIT, "cores": cpu_cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- main

def run_case(args):
    """One kernel of the path alone (for profiling): prints a small JSON line."""
    import global_attention_swa_b200 as mimo

    dev = torch.device("cuda", torch.cuda.current_device())
    T = args.seq_len
    if args.case == "prefill_backward":
        # one global layer's backward (its forward runs once, untimed)
        x = W.prefill_inputs([T], seed=1, device=dev)
        o, l = mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, 0, x.cu_seqlens, T)
        gen = torch.Generator(device=dev)
        gen.manual_seed(2)
        do = torch.randn(o.shape, generator=gen, device=dev).to(o.dtype)
        fn = lambda: mimo.mimo_attn_prefill_backward(x.q, x.k, x.v, o, l, do, x.sinks, 0,  # noqa: E731
                                                      x.cu_seqlens, T)
        work = (1664 * HQ * (T * (T + 1) // 2), 0)
    elif args.case.startswith("prefill"):
        window = SWA if args.case == "prefill_swa" else 0
        x = W.prefill_inputs([T], seed=1, device=dev)
        out = torch.empty((T, HQ, DV), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((HQ, T), dtype=torch.float32, device=dev)
        fn = lambda: mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, T,  # noqa: E731
                                             out=out, lse=lse)
        work = prefill_work(T, window)
    else:
        lengths = W.decode_b64_lengths(0)
        window, cap = (0, W.DECODE_GA_CAPACITY) if args.case == "decode_global" else (SWA, SWA)
        if args.case == "decode_global" and args.decode_cap:
            # smaller caches (for profiler captures): lengths ~U[1024, cap]
            cap = args.decode_cap
            lengths = W.lengths_uniform(0, 64, 1024, cap)
        if args.case == "decode_global_fp8":
            window, cap = 0, (args.decode_cap or W.DECODE_GA_CAPACITY)
            if args.decode_cap:
                lengths = W.lengths_uniform(0, 64, 1024, cap)
            d = W.decode_inputs_fp8(lengths, cap, window, seed=3, device=dev)
            fn = lambda: mimo.mimo_attn_decode_fp8(d.q, d.k_codes, d.v_codes, d.k_scale,  # noqa: E731
                                                   d.v_scale_kv, d.seqlens, window, d.sinks)
            work = decode_fp8_work(lengths, window, cap)
        else:
            d = W.decode_inputs(lengths, cap, window, seed=3, device=dev)
            fn = lambda: mimo.mimo_attn_decode(d.q, d.k_cache, d.v_cache, d.seqlens, window, d.sinks)  # noqa: E731
            work = decode_work(lengths, window, cap)
    flush = L2Flush(dev)
    for _ in range(args.warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    ms = []
    for _ in range(args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    mimo.mimo_attn_device_status()
    m = float(np.mean(ms)) if ms else float("nan")
    f, b = work
    print(json.dumps({"case": args.case, "seq_len": T, "ms": round(m, 4),
                      "TFLOP/s": round(f / (m * 1e-3) / 1e12, 1),
                      "GB/s": round(b / (m * 1e-3) / 1e9, 1)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the FP8-cache decode measured after the step")
    ap.add_argument("--case", choices=["step", "prefill_swa", "prefill_global", "decode_global",
                                       "decode_ring", "decode_global_fp8", "prefill_backward"],
                    default="step",
                    help="run one kernel alone (profiling); 'step' is the benchmark")
    ap.add_argument("--seq-len", type=int, default=T_PREFILL, help="prefill length for --case")
    ap.add_argument("--decode-cap", type=int, default=0,
                    help="decode_global(_fp8) --case with caches of this capacity (0: 262144)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    peaks, peak_kind = load_peaks()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, peaks, peak_kind)), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    if args.case != "step":
        run_case(args)
        return
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    res = run_ours(args, rank, world, peaks, peak_kind)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        smp = OracleSample(rows_swa=256, rows_ga=24, decode_seqs=1)
        v, s = smp.run(peaks)
        res["cpu_baseline"] = {"value": round(v, 6), "unit": UNIT, "cores": cpu_cores(),
                               "kind": "oracle", "sample": smp.sample, "seconds": round(s, 2)}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
