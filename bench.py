#!/usr/bin/env python
"""Benchmark of the HiLS attention forward on B200 through the C-ABI library.

A step is one pass of the whole hot path over one synthetic batch.  The
headline line times the full prefill forward of the 128K-token GQA workload
(B1, Hq32/Hkv8, d128, S64, k32, r32): calibration, landmark scoring, top-k
selection, fusion weights, per-chunk attention and the fused merge.  The
decode step at a 512K-token context (B1, H16, d64, k16) is timed in the same
run under "decode", and the other workloads under "configs": the tiny float32
problem, the 8K prefill, the decode of 32 sequences at 128K, and the decode at
4M tokens (with the recall of its planted needle chunks).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torch.distributed.run, one rank per GPU: every rank runs
its own independent sequence (weak scaling, no data-path collective); the
step time is the maximum over ranks.  ``--impl reference`` times the CPU
oracle (plain fp64 C) on a bounded sample of the same workload on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import hils_inputs as hi  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREFILL_KERNELS_PER_STEP = 7   # calib, score+select, bucket count, scan totals, scan, scatter, attend + merge (bf16)
# backward: bucket count, scan totals, scan, scatter; then the tensor-core path's
# delta, lm', attention, item sums, M sum, dA/dB, or the CUDA-core attention and scores
BACKWARD_KERNELS_TC = 10
BACKWARD_KERNELS_SIMT = 6
# decode: one cooperative kernel per step when every CTA fits on the GPU at once,
# else scan + attend; counted from the profiled eager steps (decode_report)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: d[k] for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- work counts
# DRAM traffic of the attention kernel from one ncu capture on prefill_16k_gqa
# (dram__bytes_read.sum + dram__bytes_write.sum = 562.5 MB + 114.6 MB for
# 15.76M (row, slot) pairs), per pair; it grows with the pairs.  Valid only
# for the kernel source it was taken on (sha256 below); otherwise the bench
# reports null.
ATTN_TRAFFIC = {"file": "chunk_sparse_long_b200/csrc/attn_tc.cu",
                "sha256": "dabe3af0a52ce023f9d3543722daa5c44a3f1d2ea727ee1a539c700fff426add",
                "bytes_per_pair": (562519040 + 114627328) / 15761408}


def attn_traffic(pairs: float):
    import hashlib
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), ATTN_TRAFFIC["file"])
    try:
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    return ATTN_TRAFFIC["bytes_per_pair"] * pairs if digest == ATTN_TRAFFIC["sha256"] else None


def prefill_counts(w: hi.Workload) -> dict:
    """Algorithmic work of one prefill step (all rows of all sequences)."""
    S, k, d, r = w.chunk_size, w.top_k, w.head_dim, w.calib_rank
    i = np.arange(w.seq_len, dtype=np.int64)
    c = i // S
    n_sel = np.minimum(k, c + 1)
    keys = (n_sel - 1) * S + (i % S + 1)
    rows = w.batch * w.n_q_heads
    att = float(rows * np.sum(4 * d * keys))                 # QK^T and PV, useful keys only
    score = float(rows * np.sum(2 * d * (c + 1)))            # q~ . landmark, causal chunks
    calib = float(rows * w.seq_len * 4 * d * r)
    el = 2 if w.dtype == hi.DT_BF16 else 4
    kv_bytes = w.batch * w.n_kv_heads * 2 * w.seq_len * d * el
    q_bytes = rows * w.seq_len * d * el
    lm_bytes = w.batch * w.n_kv_heads * ((w.seq_len + S - 1) // S) * d * el
    return {"attention_flop": att, "score_flop": score, "calib_flop": calib,
            "min_bytes": float(kv_bytes + 2 * q_bytes + lm_bytes), "pairs": float(rows * n_sel.sum())}


def decode_bytes(w: hi.Workload, step: int) -> dict:
    """Algorithmic HBM bytes of decode step ``step``: every visible landmark of
    each KV head, the selected chunks' K and V per query head, q, out, and the
    appended k/v."""
    S, k, d = w.chunk_size, w.top_k, w.head_dim
    t = w.seq_len + step
    c = t // S
    el = 2 if w.dtype == hi.DT_BF16 else 4
    lm = w.batch * (c + 1) * w.n_kv_heads * d * el
    n_sel = min(k, c + 1)
    keys = (n_sel - 1) * S + (t % S + 1)
    kv = w.batch * w.n_q_heads * keys * d * 2 * el
    small = w.batch * (2 * w.n_q_heads + 2 * w.n_kv_heads) * d * el
    return {"landmark_bytes": lm, "kv_bytes": kv, "total": lm + kv + small}


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.lines = []
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
        sel = ["-i", vis[self.dev].strip()] if len(vis) > self.dev and vis[self.dev].strip() else \
            ["-i", str(self.dev)]
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- our arm
def make_cache(hils, wl):
    w = wl["workload"]
    return hils.Cache(wl["pages"], wl["num_pages"], wl["block_table"], wl["max_chunks"],
                      wl["landmarks"], wl.get("seq_lens"))


def cfg_of(hils, w):
    return hils.HilsConfig(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk_size, w.top_k,
                           w.calib_rank, w.dtype)


def time_prefill(hils, torch, wl, steps, warmup, barrier, maxreduce):
    w = wl["workload"]
    cfg = cfg_of(hils, w)
    cache = make_cache(hils, wl)
    L = w.seq_len
    dt = torch.bfloat16 if w.dtype == hi.DT_BF16 else torch.float32
    out = torch.empty((w.batch, L, w.n_q_heads, w.head_dim), dtype=dt, device="cuda")
    nbytes = hils.workspace_size(cfg, hils.OP_PREFILL, L, wl["max_chunks"])
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        hils.prefill(cfg, wl["q"], L, 0, wl["A"], wl["B"], cache, out, None, None, ws, nbytes,
                     stream)

    for _ in range(warmup):
        step()
    hils.device_status(stream)
    hils.profile_reset()
    hils.profile_enable(True)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    hils.profile_enable(False)
    phases = hils.profile_read()
    hils.device_status(stream)
    ms = maxreduce(e0.elapsed_time(e1)) / steps
    return ms, phases, clk.summary(), (out, ws, nbytes)


def time_prefill_e2e(hils, torch, wl, steps, warmup):
    """Same step through host buffers: every step copies all of its inputs in
    from pinned host memory and its result out, inside the timed region.  The
    steps are pipelined over three streams, as a serving loop would run them:
    while step n computes, step n+1's inputs are copied in and step n-1's
    result is copied out (device inputs and outputs double-buffered; the
    host-to-device and device-to-host copies use the link's two directions at
    once).  The timed region runs from the first step's first copy in to the
    last step's copy out, so the pipeline's fill and drain are included."""
    w = wl["workload"]
    cfg = cfg_of(hils, w)
    keys = ("q", "pages", "landmarks", "block_table", "A", "B")
    host = {k: wl[k].cpu().pin_memory() for k in keys}
    dev = [{k: torch.empty_like(wl[k]) for k in keys} for _ in range(2)]
    L = w.seq_len
    out = [torch.empty_like(wl["q"]) for _ in range(2)]
    out_host = [torch.empty(out[0].shape, dtype=out[0].dtype).pin_memory() for _ in range(2)]
    nbytes = hils.workspace_size(cfg, hils.OP_PREFILL, L, wl["max_chunks"])
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    caches = [hils.Cache(d["pages"], wl["num_pages"], d["block_table"], wl["max_chunks"],
                         d["landmarks"]) for d in dev]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out[0].numel() * out[0].element_size()
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def run(n_steps):
        ev_in, ev_run, ev_out = [], [], []
        for n in range(n_steps):
            b = n % 2
            ev_in.append(torch.cuda.Event())
            ev_run.append(torch.cuda.Event())
            ev_out.append(torch.cuda.Event())
            with torch.cuda.stream(s_in):
                if n >= 2:
                    s_in.wait_event(ev_run[n - 2])     # step n-2 has read buffer b's inputs
                for k in keys:
                    dev[b][k].copy_(host[k], non_blocking=True)
                ev_in[n].record(s_in)
            s_run.wait_event(ev_in[n])
            if n >= 2:
                s_run.wait_event(ev_out[n - 2])        # buffer b's previous result is out
            d = dev[b]
            hils.prefill(cfg, d["q"], L, 0, d["A"], d["B"], caches[b], out[b], None, None, ws,
                         nbytes, s_run)
            ev_run[n].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_run[n])
                out_host[b].copy_(out[b], non_blocking=True)
                ev_out[n].record(s_out)

    run(warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_run.wait_event(e0)
    s_out.wait_event(e0)
    run(steps)
    e1.record(s_out)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, h2d, d2h


def time_decode(hils, torch, wl, warmup_steps=8, n_steps=0):
    """All decode steps of the workload, one after another (each appends its
    token).  The step is captured once as a CUDA graph (its three kernels keep
    their programmatic-launch overlap) and replayed per step: that step's
    inputs are staged into the graph's buffers and L2 is flushed before it, and
    only the replay is timed, so host launch cost never shows up as GPU time.
    A second, eager pass with per-kernel events gives the kernel split (events
    between the kernels serialise them, so that split over-counts)."""
    w = wl["workload"]
    cfg = cfg_of(hils, w)
    cache = make_cache(hils, wl)
    dt = torch.bfloat16 if w.dtype == hi.DT_BF16 else torch.float32
    nbytes = hils.workspace_size(cfg, hils.OP_DECODE, 1, wl["max_chunks"])
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=dt, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    seq0 = wl["seq_lens"].clone()
    sq = torch.empty_like(wl["q_dec"][0])
    sk = torch.empty_like(wl["k_new"][0])
    sv = torch.empty_like(wl["v_new"][0])

    def stage(s):
        sq.copy_(wl["q_dec"][s])
        sk.copy_(wl["k_new"][s])
        sv.copy_(wl["v_new"][s])

    def call(stream):
        hils.decode(cfg, sq, sk, sv, wl["A"], wl["B"], cache, out, None, None, ws, nbytes, stream)

    n = n_steps if n_steps > 0 else w.decode_steps
    # eager warm-up (also sets the kernels' shared-memory limits), then capture
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for s in range(warmup_steps):
            stage(s % n)
            call(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(torch.cuda.current_stream())
    stream = torch.cuda.current_stream()

    wl["seq_lens"].copy_(seq0)
    evs = []
    for s in range(n):
        stage(s)
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in evs]
    hils.device_status(stream)
    del graph

    # per-kernel split: eager steps with the event profiler
    wl["seq_lens"].copy_(seq0)
    hils.profile_reset()
    hils.profile_enable(True)
    for s in range(n):
        stage(s)
        flush.zero_()
        call(stream)
    torch.cuda.synchronize()
    hils.profile_enable(False)
    phases = hils.profile_read()
    hils.device_status(stream)
    wl["seq_lens"].copy_(seq0)
    return times, phases


def prefill_report(w: hi.Workload, ms: float, phases: dict, steps: int, n_ranks: int,
                   clocks: dict) -> dict:
    """Throughput and roofline of a timed prefill run.  The roofline is that of
    the dominant kernel: its algorithmic flops per launch over its average
    event-timed launch duration, against the measured dense bf16 peak (the
    burst figure when the SM clock held its maximum during the run, the
    sustained one otherwise)."""
    pk, pk_src = peaks()
    counts = prefill_counts(w)
    dom_name, (dom_ms_total, dom_launches) = max(phases.items(), key=lambda kv: kv[1][0])
    dom_ms = dom_ms_total / max(1, dom_launches)
    if dom_name.startswith("prefill.score_select"):
        work, what = counts["score_flop"], "useful landmark-scoring flop (q~ . landmark, causal chunks)"
    else:
        work, what = counts["attention_flop"], "useful attention flop (QK^T + PV over selected keys)"
    at_max = bool(clocks.get("sm_mhz")) and clocks.get("sm_max_mhz") and \
        clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"]
    peak = pk["bf16_tflops"] if at_max else pk["bf16_tflops_sustained"]
    achieved = work / (dom_ms / 1e3) / 1e12
    traffic = attn_traffic(counts["pairs"]) if dom_name == "prefill.attend_tc" else None
    bf16 = w.dtype == hi.DT_BF16
    return {
        "workload": w.name, "ms_per_step": ms,
        "tok_per_s": weak_scaling_value(w.batch * w.seq_len, n_ranks, ms),
        "kernels_ms_per_step": {k: v[0] / max(1, steps) for k, v in phases.items()},
        "useful_attention_tflops": counts["attention_flop"] / (ms / 1e3) / 1e12,
        "step_frac_of_peak": counts["attention_flop"] / (ms / 1e3) / 1e12 / peak,
        "roofline": {"bound": "tensor" if bf16 else "alu", "kernel": dom_name,
                     "achieved": achieved, "peak": peak if bf16 else None, "unit": "TFLOP/s",
                     "frac": achieved / peak if bf16 else None, "traffic": traffic,
                     "traffic_source": "ncu dram bytes scaled by (row, slot) pairs" if traffic else None,
                     "work_per_launch": work, "work": what,
                     "peak_source": (f"{pk_src} bf16 " + ("burst (SM clock at its maximum during the run)"
                                                          if at_max else "sustained"))
                     if bf16 else "float32 CUDA-core path: no tensor-core roofline"},
    }


def time_backward(hils, torch, wl, steps, warmup, barrier, maxreduce):
    """hils_prefill_backward on the workload.  The forward runs once first: its
    output and its selection (idx, w) are inputs of the backward, with a seeded
    N(0,1) dout.  Each timed step adds the gradients into the same float32
    buffers (the work does not depend on their contents)."""
    w = wl["workload"]
    cfg = cfg_of(hils, w)
    cache = make_cache(hils, wl)
    L, B, Hq, d, k = w.seq_len, w.batch, w.n_q_heads, w.head_dim, w.top_k
    dt = torch.bfloat16 if w.dtype == hi.DT_BF16 else torch.float32
    out = torch.empty((B, L, Hq, d), dtype=dt, device="cuda")
    idx = torch.empty((B * L * Hq, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((B * L * Hq, k), dtype=torch.float32, device="cuda")
    nf = hils.workspace_size(cfg, hils.OP_PREFILL, L, wl["max_chunks"])
    wsf = torch.empty(nf, dtype=torch.uint8, device="cuda")
    hils.prefill(cfg, wl["q"], L, 0, wl["A"], wl["B"], cache, out, idx, wt, wsf, nf)
    torch.cuda.synchronize()
    del wsf
    torch.cuda.empty_cache()
    dout = torch.empty_like(out)
    hi.normal_device(dout, w.seed, hi.TID_DOUT)
    dq = torch.zeros((B, L, Hq, d), dtype=torch.float32, device="cuda")
    dpages = torch.zeros(wl["pages"].shape, dtype=torch.float32, device="cuda")
    dlm = torch.zeros(wl["landmarks"].shape, dtype=torch.float32, device="cuda")
    dA = torch.zeros((d, w.calib_rank), dtype=torch.float32, device="cuda")
    dB = torch.zeros((w.calib_rank, d), dtype=torch.float32, device="cuda")
    nb = hils.workspace_size(cfg, hils.OP_PREFILL_BACKWARD, L, wl["max_chunks"])
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        hils.prefill_backward(cfg, wl["q"], L, 0, wl["A"], wl["B"], cache, idx, wt, out, dout, dq,
                              dpages, dlm, dA, dB, ws, nb, stream)

    for _ in range(warmup):
        step()
    hils.device_status(stream)
    hils.profile_reset()
    hils.profile_enable(True)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    hils.profile_enable(False)
    phases = hils.profile_read()
    hils.device_status(stream)
    return maxreduce(e0.elapsed_time(e1)) / steps, phases, clk.summary(), nb


def backward_report(w: hi.Workload, ms: float, phases: dict, steps: int, n_ranks: int,
                    clocks: dict, ws_bytes: int) -> dict:
    """Throughput and roofline of a timed backward run.  Algorithmic work: the
    six products per (row, chunk) pair over the keys visible to the row (the
    forward's QK^T and PV, recomputed, and dP, dQ, dK, dV), three times the
    forward's useful attention flop.  The roofline is that of the attention
    kernel against the measured dense bf16 peak (tensor-core path), or
    float32 CUDA cores (no tensor-core roofline)."""
    pk, pk_src = peaks()
    counts = prefill_counts(w)
    work = 3 * counts["attention_flop"]
    name = "backward.attention"
    tot, n = phases.get(name, (0.0, 0))
    att_ms = tot / max(1, n)
    tc = w.dtype == hi.DT_BF16 and w.head_dim == 128
    at_max = bool(clocks.get("sm_mhz")) and clocks.get("sm_max_mhz") and \
        clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"]
    peak = pk["bf16_tflops"] if at_max else pk["bf16_tflops_sustained"]
    achieved = work / (att_ms / 1e3) / 1e12 if att_ms > 0 else None
    return {
        "workload": w.name, "ms_per_step": ms, "steps": steps,
        "tok_per_s": weak_scaling_value(w.batch * w.seq_len, n_ranks, ms),
        "kernels_ms_per_step": {k: v[0] / max(1, steps) for k, v in phases.items()},
        "gpu_launches": (BACKWARD_KERNELS_TC if tc else BACKWARD_KERNELS_SIMT) * steps,
        "workspace_bytes": ws_bytes, "clocks": clocks,
        "roofline": {"bound": "tensor" if tc else "alu", "kernel": name,
                     "achieved": achieved, "peak": peak if tc else None, "unit": "TFLOP/s",
                     "frac": achieved / peak if (tc and achieved) else None, "traffic": None,
                     "work_per_launch": work,
                     "work": "useful flop of the six per-pair products over visible keys "
                             "(3x the forward's attention flop)",
                     "peak_source": (f"{pk_src} bf16 " + ("burst" if at_max else "sustained"))
                     if tc else "float32 CUDA-core path: no tensor-core roofline"},
    }


def decode_report(dw: hi.Workload, times: list, phases: dict, n_ranks: int, maxreduce) -> dict:
    """Step time and HBM roofline of a timed decode run: the step's algorithmic
    bytes (every visible landmark, the selected K/V, q, out and the appended
    k/v) over the graph-replayed step time, against the measured copy
    bandwidth."""
    pk, pk_src = peaks()
    us = maxreduce(statistics.mean(times)) * 1e3
    by = [decode_bytes(dw, s) for s in range(len(times))]
    tot = statistics.mean(b["total"] for b in by)
    kvb = statistics.mean(b["kv_bytes"] for b in by)
    lmb = statistics.mean(b["landmark_bytes"] for b in by)
    gbs = tot / (us / 1e6) / 1e9
    # kernels of one step, from the eager profiled pass over the same steps
    launches_per_step = round(sum(v[1] for v in phases.values()) / max(1, len(times)))
    return {
        "workload": dw.name, "us_per_step": us, "us_per_step_median": statistics.median(times) * 1e3,
        "steps": len(times), "batch": dw.batch, "context": dw.seq_len, "bytes_per_step": tot,
        "landmark_bytes": lmb, "kv_bytes": kvb,
        "kernels_us_per_step_serialized": {k: v[0] / max(1, v[1]) * 1e3 for k, v in phases.items()},
        "roofline": {"bound": "hbm", "kernel": "decode step (" + ("one kernel" if launches_per_step == 1
                                                               else "scan + attend, overlapped") + ")",
                     "achieved": gbs,
                     "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                     "traffic": None, "peak_source": f"{pk_src} HBM copy bandwidth"},
        "timing": "CUDA graph replay of one step; inputs staged and L2 flushed (256 MB write) "
                  "before it; only the replay is timed",
        "gpu_launches": launches_per_step * len(times),
        "kernels_per_step": launches_per_step,
    }


def decode_needle_recall(hils, torch, wl) -> dict:
    """Step 0 of a decode workload with planted needle chunks: the share of
    (sequence, query head) selections that hold every needle."""
    w = wl["workload"]
    cfg = cfg_of(hils, w)
    cache = make_cache(hils, wl)
    nbytes = hils.workspace_size(cfg, hils.OP_DECODE, 1, wl["max_chunks"])
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    dt = torch.bfloat16 if w.dtype == hi.DT_BF16 else torch.float32
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=dt, device="cuda")
    idx = torch.empty((w.batch, w.n_q_heads, w.top_k), dtype=torch.int32, device="cuda")
    wt = torch.empty((w.batch, w.n_q_heads, w.top_k), dtype=torch.float32, device="cuda")
    seq0 = wl["seq_lens"].clone()
    hils.decode(cfg, wl["q_dec"][0], wl["k_new"][0], wl["v_new"][0], wl["A"], wl["B"], cache, out,
                idx, wt, ws, nbytes)
    hils.device_status()
    wl["seq_lens"].copy_(seq0)
    sel = idx.cpu().numpy()
    needles = set(int(c) for c in wl["needle_chunks"])
    hit = [needles <= set(sel[b, h, 1:].tolist()) for b in range(w.batch) for h in range(w.n_q_heads)]
    return {"needles": sorted(needles), "heads_with_all_needles": int(sum(hit)),
            "heads": len(hit), "recall": sum(hit) / len(hit)}


# ----------------------------------------------------------------- oracle (CPU)
def oracle_prefill_sample(wl, budget_s: float, rng_seed: int = 0):
    """Time the CPU oracle on a sample of the prefill workload's rows for about
    ``budget_s`` seconds.  Returns (rows_done, seconds, threads, sample text)."""
    from oracle import oracle
    w = wl["workload"]
    threads = oracle.set_threads(0)
    pages = wl["pages"].cpu()
    to_np = (lambda t: t.view(__import__("torch").int16).numpy().view(np.uint16)) \
        if w.dtype == hi.DT_BF16 else (lambda t: t.numpy())
    pages_np = to_np(pages)
    lm_np = to_np(wl["landmarks"].cpu())
    bt = wl["block_table"].cpu().numpy()
    A, B = wl["A"].cpu().numpy(), wl["B"].cpu().numpy()
    oc = oracle.cfg(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk_size, w.top_k,
                    w.calib_rank, w.dtype)
    rng = np.random.default_rng(rng_seed)
    q = wl["q"]
    done, t0, batches = 0, time.perf_counter(), 0
    batch = max(threads * 4, 16)
    while True:
        pos = rng.integers(0, w.seq_len, size=batch)
        hh = rng.integers(0, w.n_q_heads, size=batch)
        bb = rng.integers(0, w.batch, size=batch)
        import torch
        ix = torch.from_numpy(np.stack([bb, pos, hh], 1)).to(q.device)
        rows = to_np(q[ix[:, 0], ix[:, 1], ix[:, 2]].cpu())
        oracle.hils_rows(oc, rows, bb, hh, pos, A, B, pages_np, bt, lm_np)
        done += batch
        batches += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    sample = (f"{done} query rows (random positions and heads, uniform over the "
              f"{w.seq_len}-token sequence) in {batches} batches; tok/s = rows/s / Hq")
    return done, el, threads, sample


# ----------------------------------------------------------------- main
def dist_ops(backend: str, device: str):
    """(barrier, maxreduce) over the initialised process group: maxreduce(x) is
    the maximum of x over all ranks (the step time of a weakly scaled run)."""
    import torch
    import torch.distributed as dist

    def barrier():
        dist.barrier()

    def maxreduce(x):
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return barrier, maxreduce


def weak_scaling_value(units_per_rank: float, n_ranks: int, step_ms_max: float) -> float:
    """Whole-job throughput: every rank processes its own units in the step,
    and the step takes as long as the slowest rank."""
    return units_per_rank * n_ranks / (step_ms_max / 1e3)


def dist_setup(torch):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
        barrier, maxreduce = dist_ops("nccl", "cuda")
        return ws, rank, barrier, maxreduce
    torch.cuda.set_device(local)
    return 1, 0, (lambda: None), (lambda x: x)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_128k_gqa")
    ap.add_argument("--decode-workload", default="decode_512k")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--skip-prefill", action="store_true",
                    help="time only the decode workload (for profiling runs)")
    ap.add_argument("--decode-steps", type=int, default=0,
                    help="timed decode steps (default: all of the workload's steps)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="time only the headline prefill and decode workloads")
    ap.add_argument("--config-decode-steps", type=int, default=64,
                    help="timed decode steps of the B=32 and 4M decode workloads")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward (hils_prefill_backward) lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    import torch
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores alone; no process group is needed
        if int(os.environ.get("RANK", "0")) != 0:
            return
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))   # the input generator
        nworld, rank = int(os.environ.get("WORLD_SIZE", "1")), 0
    else:
        nworld, rank, barrier, maxreduce = dist_setup(torch)
    w = hi.WORKLOADS[args.workload]
    counts = prefill_counts(w)
    tokens_per_rank = w.batch * w.seq_len
    metric = "HiLS prefill tok/s @128K; decode us/step @512K; % of HBM/TC roofline"
    config = {"workload": w.name, "global_batch": w.batch * nworld, "seq_len": w.seq_len,
              "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
              "chunk_size": w.chunk_size, "top_k": w.top_k, "calib_rank": w.calib_rank,
              "parallelism": f"replicas{nworld} (independent sequences)",
              "l2": "inputs larger than L2 (q 1.07 GB, K/V 0.54 GB per step)"}

    if args.impl == "reference":
        wl = hi.device_workload(w)
        budget = max(2.0, args.cpu_budget / max(1, args.steps + args.warmup) * 2)
        per = []
        for s in range(args.warmup + args.steps):
            n, el, threads, sample = oracle_prefill_sample(wl, budget, rng_seed=s)
            if s >= args.warmup:
                per.append(n / el / w.n_q_heads)
        v = statistics.median(per)
        print(json.dumps({
            "impl": "reference", "metric": metric, "value": v, "unit": "tok/s", "n_gpus": nworld,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.seq_len / v * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic N(0,1), seeded", "config": config,
            "cpu_baseline": {"value": v, "unit": "tok/s", "cores": threads, "kind": "oracle",
                             "sample": f"per step: {sample} (~{budget:.0f} s of oracle work)"},
            "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    from chunk_sparse_long_b200 import build, hils
    if rank == 0:
        build.build()
    barrier()
    hils.load()
    if args.skip_prefill:
        dw = hi.WORKLOADS[args.decode_workload]
        dwl = hi.device_workload(dw, seed_offset=rank)
        times, dph = time_decode(hils, torch, dwl, n_steps=args.decode_steps)
        if rank == 0:
            print(json.dumps({"decode_only": dw.name, "us_per_step": statistics.mean(times) * 1e3,
                              "us_per_step_median": statistics.median(times) * 1e3,
                              "kernels_us_per_step_serialized": {k: v[0] / max(1, v[1]) * 1e3
                                                                 for k, v in dph.items()}}))
        return
    wl = hi.device_workload(w, seed_offset=rank)
    torch.cuda.synchronize()
    ms, phases, clocks, _keep = time_prefill(hils, torch, wl, args.steps, args.warmup, barrier,
                                             maxreduce)
    rep = prefill_report(w, ms, phases, args.steps, nworld, clocks)
    value = rep["tok_per_s"]
    result = {
        "metric": metric, "value": value, "unit": "tok/s", "n_gpus": nworld, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic N(0,1), seeded", "config": config,
        "clocks": clocks, "roofline": rep["roofline"],
        "gpu_launches": PREFILL_KERNELS_PER_STEP * args.steps,
        "kernels_ms_per_step": rep["kernels_ms_per_step"],
        "useful_attention_tflops": rep["useful_attention_tflops"],
        "step_frac_of_peak": rep["step_frac_of_peak"],
    }
    del _keep
    if not args.no_e2e:
        e2e_ms, h2d, d2h = time_prefill_e2e(hils, torch, wl, args.steps, 1)
        e2e_ms = maxreduce(e2e_ms)
        result["e2e"] = {"value": weak_scaling_value(tokens_per_rank, nworld, e2e_ms), "unit": "tok/s",
                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                         "steps": args.steps}
    if not args.no_backward:
        bms, bph, bclk, bws = time_backward(hils, torch, wl, args.steps, args.warmup, barrier,
                                            maxreduce)
        result["backward"] = backward_report(w, bms, bph, args.steps, nworld, bclk, bws)
    del wl
    torch.cuda.empty_cache()
    configs = {}
    if not args.no_decode:
        dw = hi.WORKLOADS[args.decode_workload]
        dwl = hi.device_workload(dw, seed_offset=rank)
        times, dph = time_decode(hils, torch, dwl, n_steps=args.decode_steps)
        result["decode"] = decode_report(dw, times, dph, nworld, maxreduce)
        del dwl
        torch.cuda.empty_cache()
    if not args.no_configs:
        # the other workloads: a line each, same timing rules
        for name in ("tiny_f32", "prefill_8k"):
            pw = hi.WORKLOADS[name]
            pwl = hi.device_workload(pw, seed_offset=rank)
            pms, pph, pclk, keep = time_prefill(hils, torch, pwl, max(args.steps, 20), args.warmup,
                                                barrier, maxreduce)
            configs[name] = prefill_report(pw, pms, pph, max(args.steps, 20), nworld, pclk)
            configs[name]["clocks"] = pclk
            del keep
            if not args.no_backward and name == "prefill_8k":
                bms, bph, bclk, bws = time_backward(hils, torch, pwl, max(args.steps, 20),
                                                    args.warmup, barrier, maxreduce)
                configs[name]["backward"] = backward_report(pw, bms, bph, max(args.steps, 20),
                                                            nworld, bclk, bws)
            del pwl
            torch.cuda.empty_cache()
        for name, n in (("decode_128k_b32", args.config_decode_steps),
                        ("decode_4m", args.config_decode_steps)):
            dw = hi.WORKLOADS[name]
            dwl = hi.device_workload(dw, seed_offset=rank)
            recall = decode_needle_recall(hils, torch, dwl) if dw.needles else None
            times, dph = time_decode(hils, torch, dwl, n_steps=n)
            configs[name] = decode_report(dw, times, dph, nworld, maxreduce)
            if recall is not None:
                configs[name]["needle_recall_step0"] = recall
            del dwl
            torch.cuda.empty_cache()
        result["configs"] = configs
    if rank == 0 and nworld == 1 and not args.no_cpu_baseline:
        from oracle import oracle
        wl = hi.device_workload(w)
        n, el, threads, sample = oracle_prefill_sample(wl, args.cpu_budget)
        result["cpu_baseline"] = {"value": n / el / w.n_q_heads, "unit": "tok/s", "cores": threads,
                                  "kind": "oracle", "sample": sample}
        oracle.set_threads(1)
        n1, el1, _, sample1 = oracle_prefill_sample(wl, max(2.0, args.cpu_budget / 3), rng_seed=1)
        oracle.set_threads(threads)
        result["cpu_baseline_1core"] = {"value": n1 / el1 / w.n_q_heads, "unit": "tok/s", "cores": 1,
                                        "kind": "oracle", "sample": sample1}
    if rank == 0:
        print(json.dumps(result))
    if nworld > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
