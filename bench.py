"""Benchmark of the hybrid-precision attention hot path on B200.

One step is one pass of the whole path on a Llama-3.1-8B-shaped attention
layer with a 32768-token prompt (B=1, 32 query / 8 KV heads, head_dim 128,
5% vertical columns + 128-token window, INT4 group-32 KV):
  1. hq_probe_vertical  on the last 64 prompt queries -> vertical columns
  2. hq_prefill_attn    hybrid INT8 / bf16 causal attention over the prompt
  3. hq_pack_kv         the prompt's K / V -> hybrid INT4 + bf16 cache
  4. hq_decode_attn     the last prompt row re-attends the packed cache
The L2 cache (126 MB) is flushed before every step and again before the
decode call (the pack has just written the 47 MB cache into L2), so the
decode streams its cache from HBM.

Reported: `value` = decode-attention HBM throughput (algorithmic bytes / the
decode call's device time, CUDA events on the launching stream), plus the
prefill operator's tensor throughput, both against the measured peaks.  With
--gpus N (torchrun, one rank per GPU) every rank runs its own layer (weak
scaling, no data-path collective); timing is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hq|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_vertical_b200.synth import WORKLOADS, make_inputs, make_inputs_device  # noqa: E402

METRIC = "hybrid decode attn HBM TB/s (% of peak); hybrid prefill TFLOPS (% of peak)"
WL = WORKLOADS["llama8b_prefill_32k"]          # prompt; decode uses the same layer
NOMINAL_INT8_OVER_BF16 = 2.0                     # dense INT8 / dense bf16 (vendor ratio)


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
         "sm_max_mhz": 1965.0, "src": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        p.update({k: m[k] for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained", "sm_max_mhz")
                  if k in m})
        p["src"] = "measured"
    return p


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or None
    when the kernel's sources have changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        m = hashlib.sha256()
        for name in rec["sources"]:
            with open(os.path.join(ROOT, "kv_cache_vertical_b200", "csrc", name), "rb") as f:
                m.update(f.read())
    except (OSError, KeyError, ValueError):
        return None
    if m.hexdigest()[:16] != rec["source_sha256_16"]:
        return None
    return rec["dram_read_bytes"] + rec["dram_write_bytes"]


# ---------------------------------------------------------------------------
# Algorithmic work
# ---------------------------------------------------------------------------
def decode_bytes(B, Hq, Hkv, D, n_lo, n_hi, bits):
    """Bytes the decode must move: low codes + fp16 (s, z) + bf16 hi rows + q + fp32 out."""
    per_lo = 2 * (D * bits // 8 + (D // 32) * 4)
    per_hi = 2 * D * 2
    return B * Hkv * (n_lo * per_lo + n_hi * per_hi) + B * Hq * D * 2 + B * Hq * D * 4


def prefill_work(idx: np.ndarray, N, W, D, Hq, Hkv):
    """(INT8 ops, bf16 flops) over causal pairs only, from the actual vertical set."""
    G = Hq // Hkv
    win = sum(min(i + 1, W) for i in range(N)) if N < 4096 else (
        W * (W + 1) // 2 + (N - W) * W if N >= W else N * (N + 1) // 2)
    total = N * (N + 1) // 2
    i8 = bf = 0
    for b in range(idx.shape[0]):
        for h in range(idx.shape[1]):
            vert = int(np.maximum(0, N - W - idx[b, h].astype(np.int64)).sum())
            low = total - win - vert
            i8 += 2 * D * G * low
            bf += 2 * D * G * (total + win + vert)   # P.V over all pairs + hi QK
    return i8, bf


# ---------------------------------------------------------------------------
# Clocks during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.dev = dev_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            self.proc.wait()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9:
                    rows.append(f)
        except OSError:
            pass
        finally:
            if self.path:
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# The hq arm
# ---------------------------------------------------------------------------
def run_hq(args, rank, world, dev):
    from kv_cache_vertical_b200 import hq as H

    w = WL.replace(seed=WL.seed + rank)
    B, Hq, Hkv, D, N, W, kv = w.B, w.Hq, w.Hkv, w.D, w.L, w.window, w.k_vert
    x = make_inputs(w, pin=True)
    q_h, k_h, v_h = x["q"], x["k"], x["v"]
    q, k, v = (t.to(dev, non_blocking=True) for t in (q_h, k_h, v_h))
    stream = torch.cuda.current_stream(dev)
    idx = torch.empty(B, Hkv, kv, dtype=torch.int32, device=dev)
    out_p = torch.empty(B, Hq, N, D, dtype=torch.float32, device=dev)
    out_d = torch.empty(B, Hq, D, dtype=torch.float32, device=dev)
    cache = H.KVCache.empty(B, Hkv, N, D, W, kv, w.bits, dev, with_pos=False)
    ws_probe = H.workspace(H.hq_probe_workspace_size(B, Hq, Hkv, 64, N, D), dev)
    ws_pre = H.workspace(H.hq_prefill_workspace_size(B, Hq, Hkv, N, D, kv), dev)
    ws_pack = H.workspace(256, dev)
    ws_dec = H.workspace(H.hq_decode_workspace_size(B, Hq, Hkv, D, cache.n_lo, cache.n_hi, w.bits), dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    q_last = q[:, :, N - 1]                      # [B, Hq, D] view, stride N*D between heads
    q_dec = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    ev = {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for n in ("probe", "prefill", "pack", "decode", "step")}

    def step(qq, kk, vv, timed):
        e = ev if timed else None
        flush.zero_()
        if e: e["step"][0].record(stream)
        if e: e["probe"][0].record(stream)
        H.hq_probe_vertical(qq[:, :, N - 64:], N * D, kk, B, Hq, Hkv, 64, N, D, W, kv, 0.0, idx,
                            None, ws_probe)
        if e: e["probe"][1].record(stream)
        if e: e["prefill"][0].record(stream)
        H.hq_prefill_attn(qq, kk, vv, idx, B, Hq, Hkv, N, D, W, kv, 0.0, out_p, ws_pre)
        if e: e["prefill"][1].record(stream)
        if e: e["pack"][0].record(stream)
        H.hq_pack_kv(kk, vv, idx, B, Hkv, N, D, W, kv, w.bits, 32, cache, ws_pack)
        if e: e["pack"][1].record(stream)
        q_dec.copy_(qq[:, :, N - 1])
        flush.zero_()
        if e: e["decode"][0].record(stream)
        H.hq_decode_attn(q_dec, cache, B, Hq, Hkv, D, 0.0, out_d, None, ws_dec)
        if e: e["decode"][1].record(stream)
        if e: e["step"][1].record(stream)

    for _ in range(args.warmup):
        step(q, k, v, False)
    torch.cuda.synchronize(dev)
    acc = {n: 0.0 for n in ev}
    barrier(world)
    torch.cuda.synchronize(dev)
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(q, k, v, True)
            torch.cuda.synchronize(dev)   # per-kernel events are read back each step
            for n, (a, b) in ev.items():
                acc[n] += a.elapsed_time(b)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    total_ms = t0.elapsed_time(t1)
    per = {n: acc[n] / args.steps for n in acc}           # ms per launch
    per = {n: max_over_ranks(vv_, world, dev) for n, vv_ in per.items()}

    # e2e through the public API: host (pinned) inputs in, results back to host
    out_p_h = torch.empty(out_p.shape, dtype=out_p.dtype, pin_memory=True)
    out_d_h = torch.empty(out_d.shape, dtype=out_d.dtype, pin_memory=True)
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    e2e_steps = max(1, min(args.steps, 5))
    barrier(world)
    torch.cuda.synchronize(dev)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(e2e_steps):
        qd.copy_(q_h, non_blocking=True)
        kd.copy_(k_h, non_blocking=True)
        vd.copy_(v_h, non_blocking=True)
        step(qd, kd, vd, False)
        out_p_h.copy_(out_p, non_blocking=True)
        out_d_h.copy_(out_d, non_blocking=True)
    a1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(a0.elapsed_time(a1) / e2e_steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
    d2h = out_p.numel() * 4 + out_d.numel() * 4

    loop = decode_loop(H, w, q, k, v, q_dec, dev, stream, world)
    dconf = decode_configs(H, dev, stream, world, rank)
    graph = decode_graph(H, w, q_dec, cache, out_d, ws_dec, dev, world)
    fp8 = fp8_leg(H, w, q, k, v, idx, q_dec, dev, stream, world)
    i8_tops = int8_gemm_peak(dev)

    idx_np = idx.cpu().numpy()
    dbytes = decode_bytes(B, Hq, Hkv, D, cache.n_lo, cache.n_hi, w.bits)
    i8_ops, bf_flops = prefill_work(idx_np, N, W, D, Hq, Hkv)
    clocks = clk.summary()
    return dict(per=per, total_ms=max_over_ranks(total_ms / args.steps, world, dev), dbytes=dbytes,
                i8=i8_ops, bf=bf_flops, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, clocks=clocks,
                kpad=(kv + 63) // 64 * 64, w=w, loop=loop, fp8=fp8, i8_tops=i8_tops, graph=graph,
                idx=idx_np, dconf=dconf)


# The decode workloads timed after the steps, each on its own full-size cache.
DECODE_CONFIGS = ("llama8b_decode_32k", "batched_decode_128k_int4", "batched_decode_128k_int8",
                  "70b_decode_64k")


def decode_configs(H, dev, stream, world, rank, reps=15):
    """Decode attention alone on every decode workload of the specification,
    at full size: inputs drawn on the device (same recipe as the parity
    inputs), the vertical set from the GPU probe, the cache from the GPU
    pack; then `reps` timed calls (two untimed first), the L2 flushed before
    every call, CUDA events on the launching stream; median and best."""
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    pk = peaks()
    res = {}
    for name in DECODE_CONFIGS:
        w = WORKLOADS[name]
        x = make_inputs_device(w, dev, seed_offset=rank)
        idx = H.probe_vertical(x["q_probe"], x["k"], w.window, w.k_vert)
        cache = H.pack_kv(x["k"], x["v"], idx, w.window, w.bits, with_pos=False)
        q = x["q"]
        del x
        ws = H.workspace(H.hq_decode_workspace_size(w.B, w.Hq, w.Hkv, w.D, cache.n_lo, cache.n_hi,
                                                    w.bits), dev)
        out = torch.empty(w.B, w.Hq, w.D, dtype=torch.float32, device=dev)
        barrier(world)
        ts = []
        for i in range(reps + 2):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            H.hq_decode_attn(q, cache, w.B, w.Hq, w.Hkv, w.D, 0.0, out, None, ws)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= 2:
                ts.append(e0.elapsed_time(e1) * 1e3)
        med = max_over_ranks(float(np.median(ts)), world, dev)
        best = max_over_ranks(min(ts), world, dev)
        nb = decode_bytes(w.B, w.Hq, w.Hkv, w.D, cache.n_lo, cache.n_hi, w.bits)
        res[name] = {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "window": w.window,
                     "vertical_frac": float(w.frac), "kv_bits": w.bits,
                     "algorithmic_bytes": nb, "us_median": med, "us_best": best,
                     "gbs": nb / (med * 1e-6) / 1e9, "frac": nb / (med * 1e-6) / 1e9 / pk["hbm_gbs"],
                     "frac_of_8TBs": nb / (med * 1e-6) / 8e12}
        del cache, ws, out, q, idx
        torch.cuda.empty_cache()
    res["note"] = (f"decode alone, median of {reps} calls, L2 flushed (256 MB write) before each; "
                   "frac = algorithmic bytes / median time / measured HBM copy peak; inputs drawn "
                   "on the device (make_inputs_device)")
    return res


def decode_roofline(dconf, name, pk):
    """Roofline fields of the decode kernel on one decode workload of the
    decode_configs leg (DRAM traffic from the committed ncu record of that
    workload, or null once the kernel's sources have changed)."""
    c = dconf[name]
    return {"kernel": "decode_tma (hq_decode_attn)", "workload": name, "bound": "hbm",
            "achieved": c["gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": c["frac"],
            "traffic": profiled_traffic("decode_tma"), "algorithmic_bytes": c["algorithmic_bytes"],
            "us": c["us_median"], "peak_src": pk["src"] + " (copy bandwidth)",
            "frac_of_8TBs": c["frac_of_8TBs"]}


def decode_graph(H, w, q_dec, cache, out, ws, dev, world, n=50, reps=7):
    """The packed 32K decode as n back-to-back calls captured in one CUDA
    graph, replayed `reps` times: per-call median and best.  The 47 MB cache
    stays in the L2 between calls, so this is the call's latency floor, not
    an HBM figure.  Run at N = 1 only: a capture beside a live NCCL
    communicator is not worth the risk for an informative figure."""
    if world > 1:
        return {"skipped": "run at N = 1 only"}
    try:
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            H.hq_decode_attn(q_dec, cache, w.B, w.Hq, w.Hkv, w.D, 0.0, out, None, ws, s)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
            for _ in range(n):
                H.hq_decode_attn(q_dec, cache, w.B, w.Hq, w.Hkv, w.D, 0.0, out, None, ws, s)
        ts = []
        with torch.cuda.stream(s):            # replay() launches on the current stream
            g.replay()
            torch.cuda.synchronize(dev)
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                g.replay()
                e1.record(s)
                torch.cuda.synchronize(dev)
                ts.append(e0.elapsed_time(e1) * 1e3 / n)
        del g
        med, best, err = float(np.median(ts)), min(ts), None
    except RuntimeError as e:          # capture unsupported: report, do not fail the bench
        med, best, err = float("inf"), float("inf"), str(e).splitlines()[0][:200]
    # every rank joins the same reductions, whatever happened to its capture
    med, best = max_over_ranks(med, world, dev), max_over_ranks(best, world, dev)
    if err is not None or med == float("inf"):
        return {"error": err or "capture failed on another rank"}
    return {"calls_per_graph": n, "us_per_call_median": med, "us_per_call_best": best,
            "l2": "warm (cache fits the L2)"}


def int8_gemm_peak(dev, n=8192, reps=10):
    """INT8 tensor throughput of this GPU from a library GEMM (torch._int_mm,
    int8 x int8 -> int32, n^3, 2 n^3 ops), best of `reps` (CUDA events), run
    after everything else.  None where the library has no such GEMM."""
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        for _ in range(2):
            torch._int_mm(a, b)
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except (RuntimeError, AttributeError):
        return None


def fp8_leg(H, w, q, k, v, idx, q_dec, dev, stream, world, reps=5):
    """The FP8 (E4M3) low-bit format on the same layer and vertical set,
    after the timed steps: the prefill with an FP8 low part, and an FP8 KV
    cache (pack, then decode).  Median of `reps` calls each (two untimed
    first), the L2 flushed before every call."""
    B, Hq, Hkv, D, N, W, kv = w.B, w.Hq, w.Hkv, w.D, w.L, w.window, w.k_vert
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    out_p = torch.empty(B, Hq, N, D, dtype=torch.float32, device=dev)
    out_d = torch.empty(B, Hq, D, dtype=torch.float32, device=dev)
    ws_pre = H.workspace(H.hq_prefill_workspace_size(B, Hq, Hkv, N, D, kv), dev)
    cache = H.KVCache.empty(B, Hkv, N, D, W, kv, 8, dev, with_pos=False, fmt=H.HQ_KV_FP8)
    ws_pack = H.workspace(256, dev)
    ws_dec = H.workspace(H.hq_decode_workspace_size(B, Hq, Hkv, D, cache.n_lo, cache.n_hi, 8), dev)

    def timed(fn):
        ts = []
        for i in range(reps + 2):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= 2:
                ts.append(e0.elapsed_time(e1))
        return max_over_ranks(float(np.median(ts)), world, dev)

    barrier(world)
    pre = timed(lambda: H.hq_prefill_attn_ex(q, k, v, idx, B, Hq, Hkv, N, D, W, kv, 0.0,
                                             H.HQ_KV_FP8, out_p, ws_pre))
    pack = timed(lambda: H.hq_pack_kv(k, v, idx, B, Hkv, N, D, W, kv, 8, 32, cache, ws_pack))
    dec = timed(lambda: H.hq_decode_attn(q_dec, cache, B, Hq, Hkv, D, 0.0, out_d, None, ws_dec))
    return {"prefill_ms": pre, "pack_ms": pack, "decode_ms": dec,
            "decode_bytes": decode_bytes(B, Hq, Hkv, D, cache.n_lo, cache.n_hi, 8)}


def decode_loop(H, w, q, k, v, q_dec, dev, stream, world, T=64):
    """Token-by-token decode after a prompt of N - T tokens: per token, the
    cache maintenance call (token enters the window ring, the oldest window
    token is quantized into the low segment) and then the decode attention.
    Measured after the timed steps, L2 not flushed (consecutive tokens), all
    T tokens queued before the first runs (a sleep kernel holds the stream),
    so the times are the device's.  Two passes over the same prefix: one
    with events around every call (per-call times, each span holding one
    launch gap), one with events only around the whole loop (back to back,
    where the launches overlap the previous kernel's tail)."""
    B, Hq, Hkv, D, N, W = w.B, w.Hq, w.Hkv, w.D, w.L, w.window
    N0 = N - T
    kv0 = int(w.frac * N0)
    k0, v0 = k[:, :, :N0].contiguous(), v[:, :, :N0].contiguous()
    idx0 = torch.empty(B, Hkv, kv0, dtype=torch.int32, device=dev)
    ws_probe = H.workspace(H.hq_probe_workspace_size(B, Hq, Hkv, 64, N0, D), dev)
    H.hq_probe_vertical(q[:, :, N0 - 64:N0], N * D, k0, B, Hq, Hkv, 64, N0, D, W, kv0, 0.0, idx0,
                        None, ws_probe)
    n_lo0 = N0 - W - kv0
    cache = H.KVCache.empty(B, Hkv, N0, D, W, kv0, w.bits, dev, with_pos=False, lo_cap=n_lo0 + T)
    k_new = k[:, :, N0:].permute(2, 0, 1, 3).contiguous()      # [T, B, Hkv, D]
    v_new = v[:, :, N0:].permute(2, 0, 1, 3).contiguous()
    ws_bytes = max(H.hq_decode_workspace_size(B, Hq, Hkv, D, n_lo0 + i, cache.n_hi, w.bits)
                   for i in range(1, T + 1))
    ws = H.workspace(ws_bytes, dev)
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=dev)

    def run(per_call):
        cache.n_lo = n_lo0
        H.hq_pack_kv(k0, v0, idx0, B, Hkv, N0, D, W, kv0, w.bits, 32, cache, None)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(T)]
        barrier(world)
        torch.cuda.synchronize(dev)
        torch.cuda._sleep(40_000_000)       # ~20 ms: the host queues all T tokens meanwhile
        for i in range(T):
            e = evs[i]
            if per_call or i == 0:
                e[0].record(stream)
            H.hq_kv_append(k_new[i], v_new[i], B, Hkv, D, N0 + i, W, kv0, cache)
            cache.n_lo += 1
            if per_call:
                e[1].record(stream)
            H.hq_decode_attn(q_dec, cache, B, Hq, Hkv, D, 0.0, out, None, ws)
            if per_call or i == T - 1:
                e[2].record(stream)
        ahead = not evs[0][0].query()      # the first token had not run when the last was queued
        torch.cuda.synchronize(dev)
        tot = evs[0][0].elapsed_time(evs[-1][2]) * 1e3 / T
        if not per_call:
            return tot, ahead
        app = [e[0].elapsed_time(e[1]) * 1e3 for e in evs]
        dec = [e[1].elapsed_time(e[2]) * 1e3 for e in evs]
        return float(np.median(app)), float(np.median(dec)), tot, ahead

    app, dec, tot_ev, ahead1 = run(True)
    tot_b2b, ahead2 = run(False)
    return {"tokens": T, "context": [N0 + 1, N],
            "append_us": max_over_ranks(app, world, dev),
            "decode_us": max_over_ranks(dec, world, dev),
            "us_per_token_with_events": max_over_ranks(tot_ev, world, dev),
            "us_per_token": max_over_ranks(tot_b2b, world, dev),
            "launches_per_token": 3, "l2": "not flushed",
            "queued_ahead": bool(ahead1 and ahead2)}


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample
# ---------------------------------------------------------------------------
def oracle_decode_sample(w, heads_kv: int):
    """Time the oracle's decode over `heads_kv` KV heads of the workload."""
    import oracle
    x = make_inputs(w.replace(Hkv=heads_kv, Hq=heads_kv * w.G))
    sc = oracle.probe_scores(x["q"][:, :, w.L - 64:].contiguous(), x["k"], heads_kv)
    idx = oracle.topk(sc, w.window, w.k_vert)
    c = oracle.pack_kv(x["k"], x["v"], idx, w.window, w.bits)
    q_dec = x["q"][:, :, w.L - 1].contiguous()
    t = time.perf_counter()
    oracle.decode_attn(q_dec, c, heads_kv)
    dt = time.perf_counter() - t
    nbytes = decode_bytes(w.B, heads_kv * w.G, heads_kv, w.D, c["n_lo"], c["n_hi"], w.bits)
    return nbytes, dt, oracle.max_threads()


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w):
    nbytes, dt, cores = oracle_decode_sample(w, w.Hkv)
    return {"value": nbytes / dt / 1e12, "unit": "TB/s", "cores": cores, "kind": "oracle",
            "sample": f"oracle fp64 decode attention over the full {w.L}-token INT4 cache, "
                      f"{w.Hq} query heads (one call, {dt:.2f} s)",
            "cpu_model": cpu_model(), "nproc": os.cpu_count()}


def cpu_baseline_prefill(w, idx: np.ndarray, per_stratum: int = 32):
    """The oracle's hybrid prefill on a stratified sample of query rows (the
    first rows, rows around the window boundary, the middle and the last),
    every query head, with the GPU's vertical set; the whole-layer time is
    extrapolated by causal pairs (a row's cost grows with its key count) and
    labelled as such."""
    import oracle
    N, W = w.L, w.window
    x = make_inputs(w)
    t0 = time.perf_counter()
    quant = oracle.prefill_quant(x["q"], x["k"], idx)
    t_quant = time.perf_counter() - t0
    k = per_stratum
    rows = np.unique(np.concatenate([np.arange(k), max(W - k // 2, 0) + np.arange(k),
                                     N // 2 - k // 2 + np.arange(k), N - k + np.arange(k)]))
    rows = rows[(rows >= 0) & (rows < N)].astype(np.int32)
    t0 = time.perf_counter()
    oracle.prefill_attn(x["q"], x["k"], x["v"], idx, W, quant=quant, rows=rows)
    t_rows = time.perf_counter() - t0
    pairs_sampled = int((rows.astype(np.int64) + 1).sum())
    pairs_total = N * (N + 1) // 2
    est_s = t_quant + t_rows * pairs_total / pairs_sampled
    return {"value": est_s * 1e3, "unit": "ms (whole prefill, extrapolated)", "kind": "oracle",
            "extrapolated": True, "cores": oracle.max_threads(), "rows_sampled": int(rows.size),
            "sample_s": t_quant + t_rows,
            "sample": f"oracle fp64 hybrid prefill of {rows.size} stratified query rows x {w.Hq} "
                      f"query heads (plus the whole INT8 pre-pass); time per causal pair scaled "
                      f"to all {pairs_total} pairs"}


def run_reference(args, rank, world):
    """--impl reference: the oracle as it stands, timed on the host cores."""
    if rank != 0:
        return None
    w = WL
    vals = []
    cores = 1
    hk = 2          # bounded sample per step: 2 of the 8 KV heads
    for i in range(args.warmup + args.steps):
        nbytes, dt, cores = oracle_decode_sample(w, hk)
        if i >= args.warmup:
            vals.append((nbytes, dt))
    tb = sum(b for b, _ in vals) / sum(t for _, t in vals) / 1e12
    ms = 1e3 * sum(t for _, t in vals) / len(vals)
    cpu = {"value": tb, "unit": "TB/s", "cores": cores, "kind": "oracle",
           "sample": f"oracle fp64 decode of {hk} of {w.Hkv} KV heads ({hk * w.G} query heads) "
                     f"over the {w.L}-token INT4 cache per step",
           "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    return {"impl": "reference", "metric": METRIC, "value": tb, "unit": "TB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(w, world), "cpu_baseline": cpu,
            "e2e": {"value": tb, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def config_dict(w, world):
    return {"workload": "llama3.1-8b-shaped attention layer, 32768-token prompt: probe + hybrid "
                        "prefill + INT4 pack + decode",
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.D, "tokens": w.L,
            "window": w.window, "vertical_frac": float(w.frac), "kv_bits": w.bits,
            "group": 32, "parallelism": f"replicas x{world}",
            "l2": "flushed (256 MB write) before every step and before the decode call"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="hq", choices=["hq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if world > 1:
            torch.distributed.init_process_group("gloo", timeout=__import__("datetime").timedelta(seconds=600))
        r = run_reference(args, rank, world)
        if r is not None:
            print(json.dumps(r), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        torch.distributed.init_process_group("nccl", device_id=dev,
                                             timeout=__import__("datetime").timedelta(seconds=300))
    r = run_hq(args, rank, world, dev)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    pk = peaks()
    per = r["per"]
    w = r["w"]
    dec_tbs = r["dbytes"] / (per["decode"] * 1e-3) / 1e12
    pre_s = per["prefill"] * 1e-3
    # INT8 peak: the larger (stricter) of 2 x the measured bf16 peak and the
    # INT8 GEMM measured in this run
    i8_peak = max(pk["bf16_tflops"] * NOMINAL_INT8_OVER_BF16, r["i8_tops"] or 0.0)
    t_star = r["bf"] / (pk["bf16_tflops"] * 1e12) + r["i8"] / (i8_peak * 1e12)
    pre_tflops = (r["bf"] + r["i8"]) / pre_s / 1e12
    exps = w.Hq * w.B * w.L * (w.L + 1) // 2
    # nominal ex2 rate: 16 per SM per clock at the maximum SM clock
    mufu_peak = 16.0 * torch.cuda.get_device_properties(0).multi_processor_count * pk["sm_max_mhz"] * 1e6
    mixed_peak = (r["bf"] + r["i8"]) / t_star / 1e12
    # probe 4 (two QK passes, row stats, top-k); prefill 4 (+1 vertical
    # gather when there are vertical columns); pack 1; decode 2 (split-KV
    # kernel and the combine)
    launches_per_step = 4 + (4 + (1 if r["kpad"] > 0 else 0)) + 1 + 2
    out = {
        "metric": METRIC,
        "value": dec_tbs * world,
        "unit": "TB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": r["total_ms"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int4 KV codes -> bf16/fp16 MMA, fp32 accumulate (decode); int8 + bf16/fp16 (prefill)",
        "data": "synthetic (seeded generator: outlier channels, planted vertical lines)",
        "config": config_dict(w, world),
        # the dominant kernel of the step (about 90% of its launch time) is the prefill
        "roofline": {"kernel": "prefill_tc (hq_prefill_attn)", "bound": "tensor",
                     "achieved": pre_tflops, "peak": mixed_peak, "unit": "TFLOP/s",
                     "frac": pre_tflops / mixed_peak, "traffic": profiled_traffic("prefill_tc"),
                     "ms": per["prefill"], "roofline_ms": t_star * 1e3,
                     "int8_tops": r["i8"] / 1e12, "bf16_tflop": r["bf"] / 1e12,
                     "int8_gemm_tops_measured": r["i8_tops"],
                     # the exp is the co-bound: one per (causal pair, query head)
                     "exps": exps, "exp_rate_tps": exps / pre_s / 1e12,
                     "exp_frac_of_nominal_mufu": exps / pre_s / mufu_peak,
                     "peak_src": pk["src"] + " bf16 burst GEMM peak; INT8 = the larger of bf16 x "
                                 "nominal ratio 2 and the INT8 GEMM measured in this run "
                                 "(torch._int_mm 8192^3); peak = work-weighted mix of the two"},
        # the decode kernel's roofline on the largest decode workload of the
        # specification (70B-shaped, 2.9 GB cache: HBM-bound); the step's 32K
        # decode, whose throughput is `value`, follows as decode_step
        "decode": decode_roofline(r["dconf"], "70b_decode_64k", pk),
        "decode_step": {"kernel": "decode_tma (hq_decode_attn)", "bound": "hbm",
                        "achieved": dec_tbs * 1e3, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": dec_tbs * 1e3 / pk["hbm_gbs"], "algorithmic_bytes": r["dbytes"],
                        "us": per["decode"] * 1e3, "peak_src": pk["src"] + " (copy bandwidth)",
                        "frac_of_8TBs": dec_tbs / 8.0,
                        "note": "the 32K layer's decode inside the step (latency-bound at 47 MB)"},
        "per_call_ms": {n: per[n] for n in ("probe", "prefill", "pack", "decode")},
        "probe_frac_of_prefill": per["probe"] / per["prefill"],
        # token-by-token decode after the timed steps: cache maintenance + attention
        "decode_loop": r["loop"],
        "decode_graph": r["graph"],
        # decode alone on every decode workload of the specification (full size)
        "decode_configs": r["dconf"],
        # the FP8 (E4M3) low-bit format on the same layer, after the timed steps
        "fp8": {"prefill_ms": r["fp8"]["prefill_ms"],
                "prefill_frac": t_star * 1e3 / r["fp8"]["prefill_ms"],
                "pack_ms": r["fp8"]["pack_ms"],
                "decode_us": r["fp8"]["decode_ms"] * 1e3,
                "decode_gbs": r["fp8"]["decode_bytes"] / (r["fp8"]["decode_ms"] * 1e-3) / 1e9,
                "decode_frac": r["fp8"]["decode_bytes"] / (r["fp8"]["decode_ms"] * 1e-3) / 1e9
                / pk["hbm_gbs"],
                "note": "prefill: FP8 QK at the INT8 rate (nominal FP8 = INT8 on B200), same T*; "
                        "decode: E4M3 codes + fp16 scales, median of 5, L2 flushed"},
        "e2e": {"value": r["dbytes"] / (r["e2e_ms"] * 1e-3) / 1e12 * world, "unit": "TB/s",
                "ms_per_step": r["e2e_ms"],
                "prompt_tokens_per_s": w.B * w.L / (r["e2e_ms"] * 1e-3) * world,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "note": "value = decode bytes / whole-step time (the metric's unit); ms_per_step "
                        "and prompt_tokens_per_s are the same step: pinned-host Q/K/V copied in, "
                        "probe + prefill + pack + decode, the prefill and decode outputs copied "
                        "back"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": r["clocks"],
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
        out["cpu_baseline_prefill"] = cpu_baseline_prefill(w, r["idx"])
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
