#!/usr/bin/env python
"""Benchmark of QK4V8 attention on B200: decode KV GB/s and prefill TFLOPS.

One step is one pass of the decode hot path over one batch of the GQA decode
workload: B=32, Hq=32, Hkv=8, one query token, KV length 8192, d=128, four
outlier channels x16 in Q and K. The step is one library call,
qk4v8_attention_decode_bf16: the split-KV block-scaled tcgen05 attention over
the pre-quantized MXFP4-K / MXFP8-V cache, which MXFP4-quantizes the step's
bf16 query rows itself. With one KV split (the library's choice for this
workload) that is a single launch that also writes the bf16 output; with
more splits a merge launch follows.
`value` is the packed KV bytes streamed per second, summed over all ranks
(weak scaling: every rank runs its own copy of the workload, with no
collective on the data path).

The JSON line also carries these sub-objects:
  - roofline: the attention kernel's achieved GB/s against the measured HBM
    copy bandwidth;
  - e2e: the same step through the public API with pinned host buffers, the
    query copied in and the output copied back every step;
  - prefill: the causal GQA prefill workload B=4, Hq=32, Hkv=8, S=8192,
    quantization of Q, K and V included, in TFLOPS;
  - cpu_baseline: the CPU oracle on a bounded sample of the same decode
    workload.
`--impl reference` times the CPU oracle alone on the decode workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QK4V8 attn: prefill TFLOPS & decode KV GB/s, % of B200 roofline"
DECODE_WORKLOAD = "decode_gqa_b32_hq32_hkv8_l8192"
PREFILL_WORKLOAD = "prefill_gqa_b4_hq32_hkv8_s8192"
KV_BYTES_PER_TOKEN_HEAD = 64 + 128 + 4 + 4   # E2M1 K codes, E4M3 V codes, K and V E8M0 scales
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--splits", type=int, default=0, help="decode KV splits (0 = library default)")
    ap.add_argument("--prefill-steps", type=int, default=10)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-extra-decode", action="store_true",
                    help="skip the long-context and speculative-verify decode workloads")
    ap.add_argument("--extra-steps", type=int, default=50, help="timed steps of each extra decode workload")
    ap.add_argument("--decode-workload", default=DECODE_WORKLOAD,
                    help="decode workload of the main measurement (a profiling aid; the headline is the default)")
    ap.add_argument("--no-decode", action="store_true",
                    help="prefill only (a profiling aid): prints the prefill object alone")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running (read only)."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over the ranks (the step time of a multi-GPU run is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(bytes_per_rank_step: int, steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job throughput: the bytes every rank streamed over the slowest rank's time (weak scaling)."""
    return bytes_per_rank_step * steps * world / (elapsed_ms * 1e-3) / 1e9


def to_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


# ----------------------------------------------------------------------------- decode

def decode_kernel_name(rows: int) -> str:
    """The split-KV kernel the library launches for `rows` = (Hq / Hkv) * nq query rows per KV head."""
    if rows <= 4:
        return "qk4v8_decode_kernel<16,4,4,3,2> (swap-AB split-KV decode)"
    if rows <= 8:
        return "qk4v8_decode_kernel<16,8,8,3,2> (swap-AB split-KV decode)"
    if rows <= 16:
        return "qk4v8_decode_kernel<16,16,16,3,2> (swap-AB split-KV decode)"
    if rows <= 32:
        return "qk4v8_decode_kernel<32,32,16,6,1> (swap-AB split-KV decode)"
    if rows <= 64:
        return "qk4v8_gqa_decode_kernel (row-owner GQA decode, key tiles balanced over one CTA per SM)"
    return "qk4v8_attention_kernel<true> (128-row split-KV decode)"


def decode_launches(rows: int, splits: int) -> int:
    """Kernel launches of one qk4v8_attention_decode_bf16 call."""
    if rows <= 32:
        return 1 if splits == 1 else 2               # split kernel (+ merge)
    if rows <= 64:
        return 2 if splits == 1 else 3               # query quantize, GQA decode kernel (+ merge of cut sequences)
    return 3                                         # query quantize, 128-row split kernel, merge


def run_decode(args, world, rank):
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[args.decode_workload]
    gen = wl.generate()
    q_host = torch.from_numpy(gen["q"].view(np.int16)).view(torch.bfloat16).pin_memory()
    q = q_host.cuda()
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    kp = qk.quantize_qk(to_dev(gen["k"]), seqlens=sl)      # the cache: quantized once, outside the timing
    vp = qk.quantize_v(to_dev(gen["v"]), seqlens=sl)
    max_len = int(gen["seqlens"].max())
    splits = args.splits if args.splits > 0 else qk.decode_default_splits(wl.B, wl.Hq, wl.Hkv, wl.Sq, max_len)
    ws_bytes = qk.decode_bf16_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.Sq, splits)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device="cuda") if ws_bytes else None
    out = torch.empty((wl.B, wl.Sq, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    kv_bytes = int(gen["seqlens"].astype(np.int64).sum()) * wl.Hkv * KV_BYTES_PER_TOKEN_HEAD

    def step():
        qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=max_len, num_splits=splits, workspace=ws, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # The K timed steps run as one CUDA graph, so host launch overhead does not
    # pace the device; two events bracket the whole replay.
    rows = wl.G * wl.Sq
    launches = decode_launches(rows, splits)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(args.steps):
            step()
    graph.replay()          # untimed first replay uploads the graph
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world)
    del graph
    if launches == 1:
        # The step is exactly one launch of the attention kernel: its average
        # duration is the timed region over K (back-to-back gaps included).
        attn_avg_ms = elapsed_ms / args.steps
        attn_timing = "timed region / steps (one launch per step)"
    else:
        # Several launches per step: a second replay with an event pair (graph
        # event-record nodes) around each attention call times the kernel alone.
        ev = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in range(args.steps)]
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            cap = torch.cuda.current_stream()
            for i in range(args.steps):
                ev[i][0].record(cap)
                step()
                ev[i][1].record(cap)
        g2.replay()
        torch.cuda.synchronize()
        attn_avg_ms = statistics.fmean(a.elapsed_time(b) for a, b in ev)
        attn_timing = "event pairs around each call"
        del g2

    # e2e: the public API with host buffers; the step's query is copied in and
    # its output copied back every step.
    out_host = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.steps, 500))

    def e2e_step():
        q.copy_(q_host, non_blocking=True)
        qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=max_len, num_splits=splits, workspace=ws, out=out)
        out_host.copy_(out, non_blocking=True)

    for _ in range(min(args.warmup, 5)):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)

    return dict(wl=wl, gen=gen, kv_bytes=kv_bytes, splits=splits, elapsed_ms=elapsed_ms, attn_avg_ms=attn_avg_ms,
                launches_per_step=launches, attn_timing=attn_timing,
                clocks=clk.summary(), e2e_ms=e2e_ms, e2e_steps=e2e_steps,
                h2d=q_host.numel() * 2, d2h=out_host.numel() * 2)


def run_decode_workload(name, steps, warmup, hbm_gbs):
    """One of the other decode workloads (long context, speculative verify): one
    qk4v8_attention_decode_bf16 call per step over its pre-quantized cache."""
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[name]
    gen = wl.generate()
    lens = gen["seqlens"].astype(np.int64)
    q = to_dev(gen["q"])
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    cap = qk.round_cap(wl.Lk)
    k = to_dev(gen["k"])
    kp = qk.quantize_qk(k, cap=cap, seqlens=sl)
    del k
    v = to_dev(gen["v"])
    vp = qk.quantize_v(v, cap=cap, seqlens=sl)
    del v, gen
    max_len = int(lens.max())
    splits = qk.decode_default_splits(wl.B, wl.Hq, wl.Hkv, wl.Sq, max_len)
    ws_bytes = qk.decode_bf16_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.Sq, splits)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device="cuda") if ws_bytes else None
    out = torch.empty((wl.B, wl.Sq, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")

    def step():
        qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=max_len, num_splits=splits, workspace=ws, out=out)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(steps):
            step()
    graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    del graph
    ms = t0.elapsed_time(t1) / steps
    kv_bytes = int(lens.sum()) * wl.Hkv * KV_BYTES_PER_TOKEN_HEAD   # the packed cache each step streams
    gbs = kv_bytes / (ms * 1e-3) / 1e9
    rows = wl.G * wl.Sq
    return {
        "workload": name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "nq": wl.Sq, "kv_len_mean": float(lens.mean()),
        "kv_len_max": max_len, "kv_splits": splits, "ms_per_step": ms, "value": gbs, "unit": "GB/s",
        "tokens_per_s": wl.B * wl.Sq / (ms * 1e-3),
        "launches_per_step": decode_launches(rows, splits),
        "roofline": {"bound": "hbm", "kernel": decode_kernel_name(rows), "achieved": gbs, "peak": hbm_gbs,
                     "unit": "GB/s", "frac": gbs / hbm_gbs, "algorithmic_bytes_per_step": kv_bytes,
                     "note": "step time (all launches of the call); the split kernel dominates it"},
        "clocks": clk.summary(),
    }


# ---------------------------------------------------------------------------- prefill

def run_prefill(args):
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[PREFILL_WORKLOAD]
    gen = wl.generate()
    q, k, v = to_dev(gen["q"]), to_dev(gen["k"]), to_dev(gen["v"])
    del gen
    stream = torch.cuda.current_stream()
    qp, kp, vp = qk.quantize(q, k, v)
    out = torch.empty((wl.B, wl.Sq, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")
    row_max = torch.empty((wl.B, wl.Hq, wl.Sq), dtype=torch.float32, device="cuda")
    n = max(1, args.prefill_steps)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]

    def step(i=None):
        nonlocal qp, kp, vp
        qp, kp, vp = qk.quantize(q, k, v)
        if i is not None:
            ev[i][0].record(stream)
        qk.attention_prefill(qp, kp, vp, causal=True, out=out)
        if i is not None:
            ev[i][1].record(stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record(stream)
        for i in range(n):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    attn_ms = statistics.fmean(a.elapsed_time(b) for a, b in ev)

    # The QK^T stage alone: the same kernel built without exp, P and P.V, same tile schedule.
    for _ in range(3):
        qk.prefill_stage_qk(qp, kp, causal=True, row_max=row_max)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(n):
        qk.prefill_stage_qk(qp, kp, causal=True, row_max=row_max)
    s1.record(stream)
    torch.cuda.synchronize()
    stage_ms = s0.elapsed_time(s1) / n

    # FlashAttention-style FLOP count of causal attention: 4 * B * Hq * d * (S(S+1)/2)
    pairs = wl.Sq * (wl.Sq + 1) / 2
    flops = 4.0 * wl.B * wl.Hq * 128 * pairs
    qk_flops = flops / 2
    # Executed work: every 128 x 128 tile on or below the causal diagonal is computed in full.
    nt = (wl.Sq + 127) // 128
    tiles = wl.B * wl.Hq * nt * (nt + 1) // 2
    return dict(wl=wl, ms=ms, attn_ms=attn_ms, stage_ms=stage_ms, flops=flops, qk_flops=qk_flops, tiles=tiles,
                clocks=clk.summary())


def run_mma_peaks(kinds=(0, 1), iters=200000):
    """Tensor-pipe peak (TFLOP/s) of the attention's own MMA shapes, one CTA per SM, CUDA-event timed."""
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    stream = torch.cuda.current_stream()
    res = {}
    for kind in kinds:
        qk.mma_peak_run(kind, sms, 1000)
        torch.cuda.synchronize()
        best = 0.0
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fl = qk.mma_peak_run(kind, sms, iters)
            b.record(stream)
            torch.cuda.synchronize()
            best = max(best, fl / (a.elapsed_time(b) * 1e-3) / 1e12)
        name, m, nn, kk = qk.MMA_PEAK_SHAPES[kind]
        res[f"{name}_m{m}n{nn}k{kk}"] = best
    return res


# ------------------------------------------------------------------------ CPU oracle

def oracle_decode_sample(gen, wl, target_s: float, max_units=None):
    """Time the CPU oracle on whole (b, h_kv) units of the decode workload.

    Per unit: MXFP4 quantization of the unit's query rows and fp64 attention
    over the unit's cache, the same work as one GPU step restricted to that
    unit. The cache is quantized beforehand, as it is on the GPU path.
    Returns (kv_bytes_processed, seconds, units, threads)."""
    import oracle
    B, Hkv, G, nq, L = wl.B, wl.Hkv, wl.G, wl.Sq, wl.Lk
    done_bytes, done_s, units = 0, 0.0, 0
    b = 0
    while b < B and done_s < target_s and (max_units is None or units < max_units):
        sub = dict(q=gen["q"][b:b + 1], k=gen["k"][b:b + 1], v=gen["v"][b:b + 1], seqlens=gen["seqlens"][b:b + 1])
        kc, ks = oracle.quantize_qk(sub["k"])
        vc, vs = oracle.quantize_v(sub["v"], sub["seqlens"])
        t = time.perf_counter()
        qc, qs = oracle.quantize_qk(sub["q"])
        oracle.attention(qc, qs, kc, ks, vc, vs, sub["seqlens"], causal=True)
        done_s += time.perf_counter() - t
        done_bytes += Hkv * int(sub["seqlens"][0]) * KV_BYTES_PER_TOKEN_HEAD
        units += Hkv
        b += 1
    return done_bytes, done_s, units, oracle.num_threads()


def run_reference(args, world, rank):
    """--impl reference: the CPU oracle, as it stands, on the decode workload."""
    if rank != 0:
        return 0
    import oracle
    import synth
    wl = synth.WORKLOADS[DECODE_WORKLOAD]
    gen = wl.generate()
    # One reference step = one batch entry (8 KV heads x 8192 keys) of the workload.
    b_cycle = list(range(wl.B))
    cache = {}

    def unit(b):
        if b not in cache:
            kc, ks = oracle.quantize_qk(gen["k"][b:b + 1])
            vc, vs = oracle.quantize_v(gen["v"][b:b + 1], gen["seqlens"][b:b + 1])
            cache[b] = (kc, ks, vc, vs)
        return cache[b]

    def step(i):
        b = b_cycle[i % len(b_cycle)]
        kc, ks, vc, vs = unit(b)
        qc, qs = oracle.quantize_qk(gen["q"][b:b + 1])
        oracle.attention(qc, qs, kc, ks, vc, vs, gen["seqlens"][b:b + 1], causal=True)

    steps = max(1, args.steps)
    # Bound the whole run to a few minutes: time the first step, cap the count.
    for i in range(min(args.warmup, 2)):
        step(i)
    t = time.perf_counter()
    step(0)
    one = time.perf_counter() - t
    steps_run = max(1, min(steps, int(120.0 / max(one, 1e-3))))
    for i in range(steps_run):
        unit(b_cycle[i % len(b_cycle)])   # quantize the cache outside the timing
    t = time.perf_counter()
    for i in range(steps_run):
        step(i)
    sec = time.perf_counter() - t
    step_bytes = wl.Hkv * wl.Lk * KV_BYTES_PER_TOKEN_HEAD
    value = step_bytes * steps_run / sec / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 1, "steps": steps_run,
        "warmup": min(args.warmup, 2), "ms_per_step": sec / steps_run * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DECODE_WORKLOAD, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "nq": wl.Sq, "L": wl.Lk,
                   "d": 128, "reference_step": "one batch entry: 8 KV heads x 8192 keys, 4 query rows each"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{steps_run} steps of one batch entry each (of {wl.B})"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    if steps_run < steps:
        line["steps_requested"] = steps
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------- main

def prefill_object(args, peak_src, bf16_tf):
    p = run_prefill(args)
    peaks = run_mma_peaks()
    fp4_peak = peaks["mxf4_m128n128k64"]      # the QK^T instruction's own measured peak
    fp8_peak = peaks["mxf8f6f4_m128n144k32"]  # the P.V instruction's own measured peak
    # Roofline time of the executed MMAs: QK^T in FP4; P.V twice (P_hi and P_lo terms) in FP8 at
    # N = 144 (128 channels, the ones row that sums P, padding to a multiple of 16).
    t_roof = p["qk_flops"] / (fp4_peak * 1e12) + 2 * p["qk_flops"] * (144 / 128) / (fp8_peak * 1e12)
    attn_s = p["attn_ms"] * 1e-3
    clocks = p["clocks"]
    sm_hz = (clocks.get("sm_mhz") or 1965.0) * 1e6
    # MUFU bound: one ex2 per executed score element, 16 per clock per SM.
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    mufu_s = p["tiles"] * 128 * 128 / (16.0 * sms * sm_hz)
    return {
        "workload": PREFILL_WORKLOAD, "value": p["flops"] / (p["ms"] * 1e-3) / 1e12, "unit": "TFLOPS",
        "ms_per_step": p["ms"], "steps": args.prefill_steps, "step": "quantize Q,K,V + causal prefill attention",
        "attention_ms": p["attn_ms"], "attention_tflops": p["flops"] / attn_s / 1e12,
        "roofline": {"bound": "tensor", "kernel": "qk4v8_prefill_kernel<false>",
                     "achieved": p["flops"] / attn_s / 1e12,
                     "peak": p["flops"] / t_roof / 1e12, "unit": "TFLOPS",
                     "frac": t_roof / attn_s,
                     "peak_source": "measured tcgen05 peaks of the kernel's own MMA shapes (mma_peaks)"},
        "qk_stage": {"kernel": "qk4v8_prefill_kernel<true> (QK^T stage build)", "ms": p["stage_ms"],
                     "tflops": p["qk_flops"] / (p["stage_ms"] * 1e-3) / 1e12,
                     "frac_of_measured_fp4": p["qk_flops"] / (p["stage_ms"] * 1e-3) / 1e12 / fp4_peak,
                     "frac_of_spec_fp4_9pf": p["qk_flops"] / (p["stage_ms"] * 1e-3) / 1e12 / 9000.0},
        "mma_peaks_tflops": peaks,
        "mufu_bound_ms": mufu_s * 1e3, "mufu_frac": mufu_s / attn_s,
        "bf16_x4_fp4_nominal_tflops": bf16_tf * 4.0,
        "clocks": clocks,
    }


def main():
    args = parse_args()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, world, rank)
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200); the library has no CPU path")
    world, rank, local = dist_setup(args.gpus)
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = load_peaks()

    if args.no_decode:
        if rank == 0:
            print(json.dumps({"prefill": prefill_object(args, peak_src, bf16_tf)}), flush=True)
        return 0

    d = run_decode(args, world, rank)
    wl = d["wl"]
    steps = args.steps
    value = aggregate_gbs(d["kv_bytes"], steps, world, d["elapsed_ms"])
    ms_per_step = d["elapsed_ms"] / steps
    achieved = d["kv_bytes"] / (d["attn_avg_ms"] * 1e-3) / 1e9
    e2e_value = aggregate_gbs(d["kv_bytes"], d["e2e_steps"], world, d["e2e_ms"])

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1/e4m3 MMA, f32 softmax and accumulate",
        "data": "synthetic",
        "config": {
            "workload": args.decode_workload, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "nq": wl.Sq, "L": wl.Lk, "d": 128,
            "kv_splits": d["splits"], "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"no flush: the packed KV cache ({d['kv_bytes'] / 1e6:.0f} MB) is larger than L2 (126 MB)",
            "tokens_per_s": wl.B * wl.Sq * steps * world / (d["elapsed_ms"] * 1e-3),
        },
        "roofline": {
            "bound": "hbm", "kernel": decode_kernel_name(wl.G * wl.Sq),
            "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s", "frac": achieved / hbm_gbs,
            "peak_source": f"{peak_src} hbm_gbs", "traffic": None,
            "algorithmic_bytes_per_launch": d["kv_bytes"], "avg_launch_ms": d["attn_avg_ms"],
            "launch_timing": d["attn_timing"],
        },
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": d["h2d"], "d2h_bytes_per_step": d["d2h"],
                "steps": d["e2e_steps"]},
        "gpu_launches": d["launches_per_step"] * steps,
        "clocks": d["clocks"],
    }

    if not args.no_extra_decode and world == 1:
        line["decode_workloads"] = {}
        for name in ("decode_long_b8_hq64_hkv8_l64k_128k", "verify_b64_nq8_hq64_hkv8_l16384"):
            w = run_decode_workload(name, args.extra_steps, min(args.warmup, 5), hbm_gbs)
            line["decode_workloads"][name] = w
            line["gpu_launches"] += w["launches_per_step"] * args.extra_steps
    if not args.no_prefill:
        line["prefill"] = prefill_object(args, peak_src, bf16_tf)
        line["gpu_launches"] += 4 * args.prefill_steps

    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        nbytes, sec, units, threads = oracle_decode_sample(d["gen"], wl, args.cpu_seconds)
        line["cpu_baseline"] = {"value": nbytes / sec / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"{units} of {wl.B * wl.Hkv} (b, h_kv) units, whole batch entries, "
                                          f"{sec:.1f} s"}

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
