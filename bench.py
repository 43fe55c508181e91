#!/usr/bin/env python
"""Benchmark of QK4V8 attention on B200: decode KV GB/s and prefill TFLOPS.

One step is one pass of the decode hot path over one batch of the GQA decode
workload: B=32, Hq=32, Hkv=8, one query token, KV length 8192, d=128, four
outlier channels x16 in Q and K. The step is one library call,
qk4v8_attention_decode_bf16: the split-KV block-scaled tcgen05 attention over
the pre-quantized MXFP4-K / MXFP8-V cache, which MXFP4-quantizes the step's
bf16 query rows itself. With one KV split (the library's choice for this
workload) that is a single launch that also writes the bf16 output.
`value` is the packed KV bytes streamed per second, summed over all ranks
(weak scaling: every rank runs its own copy of the workload, with no
collective on the data path).

The JSON line also carries one flat object per other workload or measurement:
  - roofline: the headline decode kernel's achieved GB/s against the measured
    HBM copy bandwidth (and the 8 TB/s specification);
  - e2e: the headline step through the public API with pinned host buffers,
    the query copied in and the output copied back every step;
  - decode_long, verify: the long-context decode (B=8, Hq=64, L in
    [65536, 131072]) and 8-token speculative verify (B=64, Hq=64, L=16384)
    workloads, each one library call per step;
  - prefill: the causal GQA prefill workload B=4, Hq=32, Hkv=8, S=8192,
    quantization of Q, K and V included, in TFLOPS, with its QK^T-stage build
    against the measured block-scaled FP4 peak of the best MMA shape;
  - prefill_small: the causal prefill B=1, Hq=Hkv=2, S=256;
  - quantize: the MXFP4 (plain and Hadamard-rotated) and MXFP8 quantize
    kernels in HBM GB/s;
  - mma_peaks: the measured tensor-pipe peaks of the block-scaled MMA shapes;
  - cpu_baseline (and cpu_* keys in each workload object): the CPU fp64
    oracle on the machine's host cores, on the whole workload (configs 1, 2, 4, 5)
    or a stated subset (the S=8192 prefill), extrapolated linearly;
  - error keys (err_*): the GPU output against the oracle, and, as context,
    against fp64 attention over the unquantized bf16 inputs; hadamard_* keys
    give the same for Q and K quantized after their Hadamard rotation, and
    qk4v4_* keys for V in MXFP4;
  - qk4v4: the decode workloads with V in MXFP4 (the article's QK4V4
    comparison point): time, GB/s of the smaller cache, speedup;
  - paged: the headline decode over 128-token pages in random order, and the
    cost of appending a token to every sequence;
  - draft_block: 8 non-causal rows with a 1024-key sliding window over the
    verify workload's cache (the DFlash draft-block attention).
`--impl reference` times the CPU oracle alone on the headline decode workload.
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
LONG_WORKLOAD = "decode_long_b8_hq64_hkv8_l64k_128k"
VERIFY_WORKLOAD = "verify_b64_nq8_hq64_hkv8_l16384"
PREFILL_WORKLOAD = "prefill_gqa_b4_hq32_hkv8_s8192"
SMALL_PREFILL_WORKLOAD = "prefill_b1_h2_s256"
KV_BYTES_PER_TOKEN_HEAD = 64 + 128 + 4 + 4   # E2M1 K codes, E4M3 V codes, K and V E8M0 scales
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
SPEC_HBM_GBS = 8000.0      # B200 HBM3e, DGX figure
SPEC_FP4_TFLOPS = 9000.0   # dense block-scaled FP4
L2_BYTES = 126 * 2 ** 20

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a
# kernel, from its committed ncu capture; None until a capture of the kernel as
# it stands exists.
NCU_TRAFFIC = {
    DECODE_WORKLOAD: (423641088, "profiles/decode_attention_b32_hq32_hkv8_l8192.md (dram read 419.78 MB + write "
                                 "3.86 MB, qk4v8_decode_kernel<16,4,4,4,2,false>, blocked V)"),
}


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
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the CPU oracle leg (baselines and error reports)")
    ap.add_argument("--no-hadamard", action="store_true", help="skip the Hadamard-rotated runs")
    ap.add_argument("--quantize-only", action="store_true",
                    help="quantize kernels only (a profiling aid): prints the quantize object alone")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running (read only)."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.0005):
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

    def _sample(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            self.reasons |= int(get_reasons(self.h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
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
            if not self.samples:
                self._sample()

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


def headline_config(world: int) -> dict:
    """The `config` object of the headline line; both arms print the same one."""
    import synth
    wl = synth.WORKLOADS[DECODE_WORKLOAD]
    kv = wl.B * wl.Hkv * wl.Lk * KV_BYTES_PER_TOKEN_HEAD
    return {"workload": DECODE_WORKLOAD, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "nq": wl.Sq, "L": wl.Lk, "d": 128,
            "parallelism": f"dp{world}: independent replicas, no collective on the data path",
            "l2": f"no flush: the packed KV cache ({kv / 1e6:.0f} MB) is larger than L2 (126 MB)"}


def to_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def graph_time_ms(step, steps, warmup, stream):
    """Runs `step` warmup times, captures `steps` calls in one CUDA graph, replays
    it once untimed, then times one replay with events. Returns (ms per step, clocks)."""
    import torch
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(steps):
            step()
    graph.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    del graph
    return t0.elapsed_time(t1) / steps, clk.summary()


# ----------------------------------------------------------------------------- decode

def decode_kernel_name(rows: int) -> str:
    """The split-KV kernel the library launches for `rows` = (Hq / Hkv) * nq query rows per KV head."""
    if rows <= 4:
        return "qk4v8_decode_kernel<16,4,4,4,2> (swap-AB split-KV decode)"
    if rows <= 8:
        return "qk4v8_decode_kernel<16,8,8,4,2> (swap-AB split-KV decode)"
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


def rotated_decode(k_dev, q_dev, vp, sl, cap, max_len, splits, steps, warmup):
    """Q and K quantized after their Hadamard rotation, then the packed decode.
    Returns (host output [B, nq, Hq, 128], ms per step of quantize(Q) + decode)."""
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    kp_r = qk.quantize_qk(k_dev, cap=cap, seqlens=sl, hadamard=True)
    qp_r = qk.quantize_qk(q_dev, hadamard=True)
    B, nq, Hq, _ = q_dev.shape
    ws = torch.empty((max(16, qk.decode_workspace_bytes(B, Hq, nq, splits)),), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, nq, Hq, 128), dtype=torch.bfloat16, device="cuda")

    def step():
        qk.quantize_qk(q_dev, hadamard=True, out=qp_r)
        qk.attention_decode(qp_r, kp_r, vp, sl, max_seqlen=max_len, num_splits=splits, workspace=ws, out=out)

    ms, _ = graph_time_ms(step, steps, warmup, torch.cuda.current_stream())
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), ms


def run_decode(args, world, rank):
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[args.decode_workload]
    gen = wl.generate()
    q_host = torch.from_numpy(gen["q"].view(np.int16)).view(torch.bfloat16).pin_memory()
    q = q_host.cuda()
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    cap = qk.round_cap(wl.Lk)
    k = to_dev(gen["k"])
    kp = qk.quantize_qk(k, cap=cap, seqlens=sl)      # the cache: quantized once, outside the timing
    vp = qk.quantize_v(to_dev(gen["v"]), cap=cap, seqlens=sl)
    max_len = int(gen["seqlens"].max())
    # The split count from the host-side lengths (qk4v8_decode_plan_splits), as a
    # serving scheduler that knows its batch would ask for it.
    splits = args.splits if args.splits > 0 else qk.decode_plan_splits(wl.B, wl.Hq, wl.Hkv, wl.Sq, gen["seqlens"])
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
        # event-record nodes) around each attention call times the call alone.
        ev = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in range(args.steps)]
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            cap_s = torch.cuda.current_stream()
            for i in range(args.steps):
                ev[i][0].record(cap_s)
                step()
                ev[i][1].record(cap_s)
        g2.replay()
        torch.cuda.synchronize()
        attn_avg_ms = statistics.fmean(a.elapsed_time(b) for a, b in ev)
        attn_timing = "event pairs around each call"
        del g2

    # e2e: the public API with host buffers; every step copies its query in from
    # pinned host memory and its output back, pipelined the way a serving loop
    # runs it: step i's upload and step i-1's download overlap step i's kernel
    # (two device buffers each for the query and the output, one stream per
    # copy direction, events for the reuse hazards). All copies of all steps lie
    # inside the timed region.
    out_host = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.steps, 500))
    q_dev = [torch.empty_like(q), torch.empty_like(q)]
    out_dev = [torch.empty_like(out), torch.empty_like(out)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        cs = torch.cuda.current_stream()   # the capturing stream under a graph capture
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_k = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        start = torch.cuda.Event()
        start.record(cs)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(n):
            j = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_k[i - 2])        # kernel i-2 has read q_dev[j]
                q_dev[j].copy_(q_host, non_blocking=True)
                ev_in[i].record(s_in)
            cs.wait_event(ev_in[i])
            if i >= 2:
                cs.wait_event(ev_out[i - 2])            # out_dev[j] of step i-2 is on the host
            qk.attention_decode_bf16(q_dev[j], kp, vp, sl, max_seqlen=max_len, num_splits=splits, workspace=ws,
                                     out=out_dev[j])
            ev_k[i].record(cs)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_k[i])
                out_host.copy_(out_dev[j], non_blocking=True)
                ev_out[i].record(s_out)
        cs.wait_event(ev_out[n - 1])                    # the last download ends the run

    e2e_run(min(args.warmup, 5))
    torch.cuda.synchronize()
    # The K steps' calls and copies are captured in one CUDA graph (the copy
    # streams fork from and join the capturing stream), so host launch overhead
    # does not pace them; the replay runs every copy and kernel again.
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph):
        e2e_run(e2e_steps)
    e2e_graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    del e2e_graph
    out_np = out.float().cpu().numpy()

    rot = None
    if world == 1 and not args.no_hadamard:
        rot = rotated_decode(k, q, vp, sl, cap, max_len, splits, 50, 3)
    del k
    return dict(wl=wl, gen=gen, kv_bytes=kv_bytes, splits=splits, elapsed_ms=elapsed_ms, attn_avg_ms=attn_avg_ms,
                launches_per_step=launches, attn_timing=attn_timing,
                clocks=clk.summary(), e2e_ms=e2e_ms, e2e_steps=e2e_steps,
                h2d=q_host.numel() * 2, d2h=out_host.numel() * 2, out=out_np, rot=rot)


def run_decode_workload(name, steps, warmup, hbm_gbs, hadamard):
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
    if not hadamard:
        del k
    v = to_dev(gen["v"])
    vp = qk.quantize_v(v, cap=cap, seqlens=sl)
    del v
    max_len = int(lens.max())
    splits = qk.decode_plan_splits(wl.B, wl.Hq, wl.Hkv, wl.Sq, gen["seqlens"])
    ws_bytes = qk.decode_bf16_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.Sq, splits)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device="cuda") if ws_bytes else None
    out = torch.empty((wl.B, wl.Sq, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")

    def step():
        qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=max_len, num_splits=splits, workspace=ws, out=out)

    ms, clocks = graph_time_ms(step, steps, warmup, torch.cuda.current_stream())
    out_np = out.float().cpu().numpy()
    rot = None
    if hadamard:
        del kp
        rot = rotated_decode(k, q, vp, sl, cap, max_len, splits, steps, 3)
        del k
    kv_bytes = int(lens.sum()) * wl.Hkv * KV_BYTES_PER_TOKEN_HEAD   # the packed cache each step streams
    gbs = kv_bytes / (ms * 1e-3) / 1e9
    rows = wl.G * wl.Sq
    res = {
        "workload": name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "nq": wl.Sq, "kv_len_mean": float(lens.mean()),
        "kv_len_max": max_len, "kv_splits": splits, "ms_per_step": ms, "steps": steps, "value": gbs,
        "unit": "GB/s", "tokens_per_s": wl.B * wl.Sq / (ms * 1e-3),
        "launches_per_step": decode_launches(rows, splits), "kernel": decode_kernel_name(rows),
        "roofline_bound": "hbm", "algorithmic_bytes_per_step": kv_bytes, "roofline_peak_gbs": hbm_gbs,
        "roofline_frac": gbs / hbm_gbs, "roofline_frac_of_spec_8tbs": gbs / SPEC_HBM_GBS,
        "roofline_timing": "step time (all launches of the call); the split kernel dominates it",
        "clocks_sm_mhz": clocks["sm_mhz"], "clocks_reasons": ",".join(clocks["reasons"]) or "none",
    }
    if rot is not None:
        res["hadamard_ms_per_step"] = rot[1]
        res["hadamard_step"] = "quantize_qk_hadamard(Q) + qk4v8_attention_decode over the rotated K cache"
    return dict(res=res, gen=gen, out=out_np, rot=None if rot is None else rot[0], wl=wl)


KV4_BYTES_PER_TOKEN_HEAD = 64 + 64 + 4 + 4   # QK4V4: E2M1 K and V codes, K and V E8M0 scales


def run_decode_v4(name, gen, steps, hbm_gbs):
    """QK4V4 (V in MXFP4) on a decode workload: the bf16-query decode step over an
    MXFP4-K / MXFP4-V cache, timed like the QK4V8 step."""
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[name]
    lens = gen["seqlens"].astype(np.int64)
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    cap = qk.round_cap(wl.Lk)
    kp = qk.quantize_qk(to_dev(gen["k"]), cap=cap, seqlens=sl)
    vp = qk.quantize_v4(to_dev(gen["v"]), cap=cap, seqlens=sl)
    q = to_dev(gen["q"])
    max_len = int(lens.max())
    splits = qk.decode_plan_splits(wl.B, wl.Hq, wl.Hkv, wl.Sq, gen["seqlens"])
    ws = torch.empty((max(16, qk.decode_bf16_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.Sq, splits)),),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.B, wl.Sq, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")

    def step():
        qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=max_len, num_splits=splits, workspace=ws, out=out)

    ms, _ = graph_time_ms(step, steps, 3, torch.cuda.current_stream())
    kv_bytes = int(lens.sum()) * wl.Hkv * KV4_BYTES_PER_TOKEN_HEAD
    gbs = kv_bytes / (ms * 1e-3) / 1e9
    return dict(ms=ms, gbs=gbs, frac=gbs / hbm_gbs, kv_bytes=kv_bytes, out=out.float().cpu().numpy())


def run_paged(gen, steps, hbm_gbs):
    """The headline decode over a paged cache: the packed cache copied into 128-token
    pages in a random page order, one qk4v8_attention_decode_bf16_paged call per
    step; plus the cost of appending one token to every sequence."""
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[DECODE_WORKLOAD]
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    max_pages = wl.Lk // 128 + 1
    k, v, q = to_dev(gen["k"]), to_dev(gen["v"]), to_dev(gen["q"])
    kp = qk.quantize_qk(k, cap=max_pages * 128, seqlens=sl)
    vp = qk.quantize_v(v, cap=max_pages * 128, seqlens=sl)
    num_pages = wl.B * max_pages
    perm = np.random.default_rng(0).permutation(num_pages).astype(np.int32).reshape(wl.B, max_pages)
    cache = qk.paged_kv(wl.B, wl.Hkv, num_pages, torch.from_numpy(perm))
    idx = cache.block_table.long()
    for i in range(max_pages):
        pages = idx[:, i]
        cache.k_codes[pages] = kp.codes[:, :, i * 128:(i + 1) * 128]
        cache.k_scales[pages] = kp.scales[:, :, i]
        cache.v_codes[pages] = vp.codes[:, :, i]
        cache.v_scales[pages] = vp.scales[:, :, i]
    cache.seqlens.copy_(sl)
    # The staging buffer holds the open V group (none: 8192 is a multiple of 32).
    out = torch.empty((wl.B, 1, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")
    ref = qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=wl.Lk)

    def step():
        qk.attention_decode_bf16_paged(q, cache, max_seqlen=wl.Lk, out=out)

    ms, _ = graph_time_ms(step, steps, 3, torch.cuda.current_stream())
    torch.cuda.synchronize()
    equal = bool(torch.equal(out, ref))
    kv_bytes = wl.B * wl.Hkv * wl.Lk * KV_BYTES_PER_TOKEN_HEAD
    # Append: one new token per sequence, 32 calls from Python, then 32 more as
    # one CUDA graph (the last page has room for 128 tokens).
    knew = k[:, :1].contiguous()
    vnew = v[:, :1].contiguous()
    n_app = 32
    stream = torch.cuda.current_stream()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(n_app):
        qk.kv_append(cache, knew, vnew)
    a1.record(stream)
    torch.cuda.synchronize()
    app_us = a0.elapsed_time(a1) / n_app * 1e3
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n_app):
            qk.kv_append(cache, knew, vnew)
    torch.cuda.synchronize()
    a0.record(stream)
    g.replay()
    a1.record(stream)
    torch.cuda.synchronize()
    app_graph_us = a0.elapsed_time(a1) / n_app * 1e3
    del g
    gbs = kv_bytes / (ms * 1e-3) / 1e9
    return {"workload": DECODE_WORKLOAD + " (paged, 128-token pages in random order)", "ms_per_step": ms,
            "value": gbs, "unit": "GB/s", "roofline_frac": gbs / hbm_gbs, "steps": steps,
            "kernel": "qk4v8_decode_kernel<16,4,4,4,2,true> (paged instance)",
            "output_equals_contiguous": equal, "append_us_per_call": app_us, "append_us_per_call_graph": app_graph_us,
            "append_call": "qk4v8_kv_append of 1 token to 32 sequences x 8 KV heads: the fused append kernel and "
                           "the in-place length update (2 launches); per call from Python, and inside a CUDA graph"}


def run_draft_block(gen, hbm_gbs, window=1024, reps=20):
    """Draft-block attention on the verify workload's cache: the 8 block rows see
    the last `window` keys before the block and the block, non-causal. Its
    working set (the window's tiles, about 110 MB) fits in L2, so L2 is flushed
    before every timed step and each step is timed alone."""
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[VERIFY_WORKLOAD]
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    cap = qk.round_cap(wl.Lk)
    kp = qk.quantize_qk(to_dev(gen["k"]), cap=cap, seqlens=sl)
    vp = qk.quantize_v(to_dev(gen["v"]), cap=cap, seqlens=sl)
    q = to_dev(gen["q"])
    out = torch.empty((wl.B, wl.Sq, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")
    splits = qk.decode_default_splits(wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.Lk, window)
    ws = torch.empty((max(16, qk.decode_bf16_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.Sq, splits)),),
                     dtype=torch.uint8, device="cuda")
    # 1 GiB: larger than L2, and its write (~160 us) outlasts the host's enqueue of
    # the timed launches, so the start event fires when the device reaches them.
    flush = torch.empty((1024 * 2 ** 20,), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=wl.Lk, causal_in_block=False, window=window,
                                 num_splits=splits, workspace=ws, out=out)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    lens = gen["seqlens"].astype(np.int64)
    lo = np.maximum(0, lens - wl.Sq - window)
    vis_bytes = int((lens - lo).sum()) * wl.Hkv * KV_BYTES_PER_TOKEN_HEAD
    gbs = vis_bytes / (ms * 1e-3) / 1e9
    return dict(res={"workload": f"draft block on {VERIFY_WORKLOAD}: 8 non-causal rows, window {window}",
                     "ms_per_step": ms, "value": gbs, "unit": "GB/s", "roofline_frac": gbs / hbm_gbs,
                     "visible_kv_bytes": vis_bytes, "kv_splits": splits, "steps": reps,
                     "l2": "flushed (1 GiB write) before each timed step",
                     "tokens_per_s": wl.B * wl.Sq / (ms * 1e-3)},
                out=out.float().cpu().numpy(), window=window)


# ---------------------------------------------------------------------------- prefill

PREFILL_SUBSET_HEADS = list(range(0, 32, 4))   # (b = 0, one query head per KV head): the CPU subset


def run_prefill(args, hadamard):
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[PREFILL_WORKLOAD]
    gen = wl.generate()
    q, k, v = to_dev(gen["q"]), to_dev(gen["k"]), to_dev(gen["v"])
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
    out_sub = out[0][:, PREFILL_SUBSET_HEADS].float().cpu().numpy()      # [S, 8, 128]

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

    rot_sub, rot_ms = None, None
    if hadamard:
        def rstep():
            qr, kr, vr = qk.quantize(q, k, v, hadamard=True)
            qk.attention_prefill(qr, kr, vr, causal=True, out=out)

        for _ in range(2):
            rstep()
        torch.cuda.synchronize()
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        for _ in range(n):
            rstep()
        r1.record(stream)
        torch.cuda.synchronize()
        rot_ms = r0.elapsed_time(r1) / n
        rot_sub = out[0][:, PREFILL_SUBSET_HEADS].float().cpu().numpy()

    # FlashAttention-style FLOP count of causal attention: 4 * B * Hq * d * (S(S+1)/2)
    pairs = wl.Sq * (wl.Sq + 1) / 2
    flops = 4.0 * wl.B * wl.Hq * 128 * pairs
    # Executed work: every 128 x 128 tile on or below the causal diagonal is computed in full.
    nt = (wl.Sq + 127) // 128
    tiles = wl.B * wl.Hq * nt * (nt + 1) // 2
    return dict(wl=wl, gen=gen, ms=ms, attn_ms=attn_ms, stage_ms=stage_ms, flops=flops, qk_flops=flops / 2,
                tiles=tiles, clocks=clk.summary(), out_sub=out_sub, rot_sub=rot_sub, rot_ms=rot_ms)


def run_prefill_small(steps=200):
    """The causal prefill B=1, Hq=Hkv=2, S=256: quantize Q, K, V + attention per step."""
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[SMALL_PREFILL_WORKLOAD]
    gen = wl.generate()
    q, k, v = to_dev(gen["q"]), to_dev(gen["k"]), to_dev(gen["v"])
    out = torch.empty((wl.B, wl.Sq, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")
    qp, kp, vp = qk.quantize(q, k, v)

    # One graph of library calls on fixed output buffers: quantize Q, K, V, attention.
    def step_fixed():
        qk.quantize_qk(q, out=qp)
        qk.quantize_qk(k, out=kp)
        qk.quantize_v(v, out=vp)
        qk.attention_prefill(qp, kp, vp, causal=True, out=out)

    ms, clocks = graph_time_ms(step_fixed, steps, 5, torch.cuda.current_stream())
    pairs = wl.Sq * (wl.Sq + 1) / 2
    flops = 4.0 * wl.B * wl.Hq * 128 * pairs
    res = {"workload": SMALL_PREFILL_WORKLOAD, "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOPS",
           "ms_per_step": ms, "steps": steps, "launches_per_step": 4,
           "step": "quantize Q, K, V + causal prefill attention (latency-bound; no roofline fraction)",
           "clocks_sm_mhz": clocks["sm_mhz"]}
    return dict(res=res, gen=gen, out=out.float().cpu().numpy(), wl=wl, flops=flops)


def run_quantize_kernels(hbm_gbs, gen, reps=10):
    """HBM throughput of the quantize kernels on the S=8192 prefill workload's
    tensors (`gen`); L2 is flushed (a 1 GiB write) before every timed launch."""
    import torch
    import bit_quantized_attention_qk4v8_b200 as qk
    import synth
    wl = synth.WORKLOADS[PREFILL_WORKLOAD]
    q, k, v = to_dev(gen["q"]), to_dev(gen["k"]), to_dev(gen["v"])
    # 1 GiB: larger than L2, and its write (~160 us) outlasts the host's enqueue of
    # the timed launches, so the start event fires when the device reaches them.
    flush = torch.empty((1024 * 2 ** 20,), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    qp = qk.quantize_qk(q)
    kp = qk.quantize_qk(k)
    vp = qk.quantize_v(v)
    cases = [
        ("quantize_qk_q", "quantize_qk_kernel<false> (Q)", lambda: qk.quantize_qk(q, out=qp),
         wl.B * wl.Sq * wl.Hq * (256 + 68)),
        ("quantize_qk_hadamard_q", "quantize_qk_kernel<true> (Q, rotated)",
         lambda: qk.quantize_qk(q, out=qp, hadamard=True), wl.B * wl.Sq * wl.Hq * (256 + 68)),
        ("quantize_qk_k", "quantize_qk_kernel<false> (K)", lambda: qk.quantize_qk(k, out=kp),
         wl.B * wl.Sq * wl.Hkv * (256 + 68)),
        ("quantize_v", "quantize_v_kernel (V)", lambda: qk.quantize_v(v, out=vp),
         wl.B * wl.Sq * wl.Hkv * (256 + 132)),
    ]
    res = {"workload": PREFILL_WORKLOAD, "unit": "GB/s", "peak_gbs": hbm_gbs,
           "bytes": "algorithmic: 256 B bf16 read + 64 B codes + 4 B scales written per Q/K token-head row; "
                    "256 B read + 128 B codes + 4 B scales per V token-head",
           "l2": "flushed (1 GiB write) before each timed launch"}
    for key, kname, fn, nbytes in cases:
        fn()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[f"{key}_us"] = ms * 1e3
        res[f"{key}_gbs"] = gbs
        res[f"{key}_frac"] = gbs / hbm_gbs
        res[f"{key}_frac_of_spec_8tbs"] = gbs / SPEC_HBM_GBS
        res[f"{key}_bytes"] = nbytes
        res[f"{key}_kernel"] = kname
    return res


def run_mma_peaks(kinds=(0, 1, 2, 3), iters=200000):
    """Tensor-pipe peak (TFLOP/s) of block-scaled MMA shapes, one CTA per SM, CUDA-event timed."""
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


def prefill_object(p, peaks):
    """Flat summary of the S=8192 prefill run against the measured MMA peaks."""
    import torch
    fp4_own = peaks["mxf4_m128n128k64"]       # the QK^T instruction's own shape
    fp8_own = peaks["mxf8f6f4_m128n144k32"]   # the P.V instruction's own shape
    fp4_best = max(v for k, v in peaks.items() if k.startswith("mxf4"))
    fp8_best = max(v for k, v in peaks.items() if k.startswith("mxf8"))
    best_fp4_shape = max((v, k) for k, v in peaks.items() if k.startswith("mxf4"))[1]
    # Roofline time of the executed MMAs: QK^T in FP4; P.V twice (P_hi and P_lo terms) in FP8 at
    # N = 144 (128 channels, the ones row that sums P, padding to a multiple of 16).
    t_own = p["qk_flops"] / (fp4_own * 1e12) + 2 * p["qk_flops"] * (144 / 128) / (fp8_own * 1e12)
    t_best = p["qk_flops"] / (fp4_best * 1e12) + 2 * p["qk_flops"] / (fp8_best * 1e12)
    attn_s = p["attn_ms"] * 1e-3
    clocks = p["clocks"]
    sm_hz = (clocks.get("sm_mhz") or 1965.0) * 1e6
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    mufu_s = p["tiles"] * 128 * 128 / (16.0 * sms * sm_hz)   # one ex2 per executed score, 16 per clock per SM
    stage_tf = p["qk_flops"] / (p["stage_ms"] * 1e-3) / 1e12
    res = {
        "workload": PREFILL_WORKLOAD, "value": p["flops"] / (p["ms"] * 1e-3) / 1e12, "unit": "TFLOPS",
        "ms_per_step": p["ms"], "steps": p.get("steps"),
        "step": "quantize Q,K,V + causal prefill attention (FlashAttention FLOP count 2.199e12)",
        "launches_per_step": 4,
        "attention_ms": p["attn_ms"], "attention_tflops": p["flops"] / attn_s / 1e12,
        "kernel": "qk4v8_prefill_kernel<false>", "roofline_bound": "tensor",
        "roofline_frac": t_best / attn_s,
        "roofline_peak_tflops": p["flops"] / t_best / 1e12,
        "roofline_peak_source": "measured tcgen05 peaks of the fastest mxf4 and mxf8f6f4 shapes (mma_peaks)",
        "roofline_frac_own_shapes": t_own / attn_s,
        "qk_stage_kernel": "qk4v8_prefill_kernel<true> (QK^T stage build)",
        "qk_stage_ms": p["stage_ms"], "qk_stage_tflops": stage_tf,
        "qk_stage_frac_of_best_fp4": stage_tf / fp4_best, "qk_stage_best_fp4_shape": best_fp4_shape,
        "qk_stage_frac_of_n128_fp4": stage_tf / fp4_own,
        "qk_stage_frac_of_spec_fp4_9pf": stage_tf / SPEC_FP4_TFLOPS,
        "mufu_bound_ms": mufu_s * 1e3, "mufu_frac": mufu_s / attn_s,
        "clocks_sm_mhz": clocks["sm_mhz"], "clocks_reasons": ",".join(clocks["reasons"]) or "none",
    }
    if p.get("rot_ms") is not None:
        res["hadamard_ms_per_step"] = p["rot_ms"]
        res["hadamard_step"] = "quantize (Q, K rotated) + causal prefill attention"
    return res


# ------------------------------------------------------------------------ CPU oracle
# Everything below runs the CPU oracle: the baselines (timed on the host cores)
# and the error reports. It is the benchmark's cpu_baseline leg.

def _errs(got, ref, prefix):
    d = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    return {f"{prefix}_max_abs": float(d.max()), f"{prefix}_mean_abs": float(d.mean())}


def cpu_decode_leg(gen, wl, out_gpu, rot_gpu, v4_gpu=None):
    """Oracle on the whole decode workload (cache pre-quantized untimed, as on the
    GPU; Q quantize + attention timed), the GPU output's error against it, and
    the context errors against unquantized attention on three batch entries."""
    import oracle
    kc, ks = oracle.quantize_qk(gen["k"])
    vc, vs = oracle.quantize_v(gen["v"], gen["seqlens"])
    t = time.perf_counter()
    qc, qs = oracle.quantize_qk(gen["q"])
    ref, _ = oracle.attention(qc, qs, kc, ks, vc, vs, gen["seqlens"], causal=True)
    sec = time.perf_counter() - t
    del kc, ks, vc, vs
    kv_bytes = int(gen["seqlens"].astype(np.int64).sum()) * wl.Hkv * KV_BYTES_PER_TOKEN_HEAD
    res = {"cpu_value": kv_bytes / sec / 1e9, "cpu_unit": "GB/s", "cpu_cores": oracle.num_threads(),
           "cpu_kind": "oracle", "cpu_seconds": sec,
           "cpu_sample": f"whole workload ({wl.B} sequences): Q quantize + fp64 attention; cache quantized untimed"}
    res.update(_errs(out_gpu, ref, "err_vs_oracle"))
    bs = sorted({0, wl.B // 2, wl.B - 1})
    got, orc, bf, rot = [], [], [], []
    for b in bs:
        one = slice(b, b + 1)
        r, _ = oracle.attention_ref(gen["q"][one], gen["k"][one], gen["v"][one], gen["seqlens"][one], causal=True)
        bf.append(r[0])
        got.append(out_gpu[b])
        orc.append(ref[b])
        if rot_gpu is not None:
            rot.append(rot_gpu[b])
    bf = np.stack(bf)
    res.update(_errs(np.stack(got), bf, "err_vs_bf16"))
    res.update(_errs(np.stack(orc), bf, "oracle_err_vs_bf16"))
    res["err_bf16_rows"] = f"batch entries {bs}, every head and query token"
    if rot_gpu is not None:
        rorc = []
        for b in bs:
            one = slice(b, b + 1)
            rqc, rqs = oracle.quantize_qk_hadamard(gen["q"][one])
            rkc, rks = oracle.quantize_qk_hadamard(gen["k"][one], gen["seqlens"][one])
            rvc, rvs = oracle.quantize_v(gen["v"][one], gen["seqlens"][one])
            o, _ = oracle.attention(rqc, rqs, rkc, rks, rvc, rvs, gen["seqlens"][one], causal=True)
            rorc.append(o[0])
        res.update(_errs(np.stack(rot), np.stack(rorc), "hadamard_err_vs_oracle"))
        res.update(_errs(np.stack(rot), bf, "hadamard_err_vs_bf16"))
    if v4_gpu is not None:
        vorc = []
        for b in bs:
            one = slice(b, b + 1)
            sub = dict(q=gen["q"][one], k=gen["k"][one], v=gen["v"][one], seqlens=gen["seqlens"][one])
            oz = oracle.quantize_workload(sub, v_fmt=oracle.E2M1)
            o, _ = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], sub["seqlens"],
                                    causal=True, v_fmt=oracle.E2M1)
            vorc.append(o[0])
        got4 = np.stack([v4_gpu[b] for b in bs])
        res.update(_errs(got4, np.stack(vorc), "qk4v4_err_vs_oracle"))
        res.update(_errs(got4, bf, "qk4v4_err_vs_bf16"))
    return res


def cpu_draft_block_leg(gen, wl, out_gpu, window):
    """Error of the draft-block (window) output against the windowed oracle and the
    windowed unquantized reference, on three batch entries."""
    import oracle
    bs = sorted({0, wl.B // 2, wl.B - 1})
    got, orc, bf = [], [], []
    for b in bs:
        one = slice(b, b + 1)
        sub = dict(q=gen["q"][one], k=gen["k"][one], v=gen["v"][one], seqlens=gen["seqlens"][one])
        oz = oracle.quantize_workload(sub)
        o, _ = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], sub["seqlens"],
                                causal=False, window=window)
        r, _ = oracle.attention_ref(sub["q"], sub["k"], sub["v"], sub["seqlens"], causal=False, window=window)
        got.append(out_gpu[b])
        orc.append(o[0])
        bf.append(r[0])
    res = _errs(np.stack(got), np.stack(orc), "err_vs_oracle")
    res.update(_errs(np.stack(got), np.stack(bf), "err_vs_bf16"))
    res["err_rows"] = f"batch entries {bs}, every head and block row"
    return res


def cpu_prefill_leg(p):
    """Oracle on a subset of the S=8192 prefill (batch entry 0, one query head per
    KV head: 8 of the 128 (b, h_q) pairs), extrapolated linearly: the quantize of
    Q, K, V of entry 0 times B, the attention of the subset times 16."""
    import oracle
    wl, gen = p["wl"], p["gen"]
    one = slice(0, 1)
    t = time.perf_counter()
    qc, qs = oracle.quantize_qk(gen["q"][one])
    kc, ks = oracle.quantize_qk(gen["k"][one])
    vc, vs = oracle.quantize_v(gen["v"][one], gen["seqlens"][one])
    t_quant = time.perf_counter() - t
    S = wl.Sq
    sel = np.array([(0, h, i) for h in PREFILL_SUBSET_HEADS for i in range(S)], dtype=np.int32)
    t = time.perf_counter()
    ref, _ = oracle.attention(qc, qs, kc, ks, vc, vs, gen["seqlens"][one], causal=True, sel=sel)
    t_attn = time.perf_counter() - t
    frac = len(PREFILL_SUBSET_HEADS) / (wl.B * wl.Hq)
    sec = t_quant * wl.B + t_attn / frac
    res = {"cpu_value": p["flops"] / sec / 1e12, "cpu_unit": "TFLOPS", "cpu_cores": oracle.num_threads(),
           "cpu_kind": "oracle", "cpu_seconds_measured": t_quant + t_attn, "cpu_seconds_extrapolated": sec,
           "cpu_sample": f"batch entry 0, query heads {PREFILL_SUBSET_HEADS[0]}..{PREFILL_SUBSET_HEADS[-1]} step "
                         f"4 (8 of 128 (b, h_q) pairs, all {S} rows): attention x16, quantize of entry 0 x{wl.B}; "
                         "extrapolated linearly"}
    got = np.transpose(p["out_sub"], (1, 0, 2)).reshape(-1, 128)     # [h, i] order like sel
    res.update(_errs(got, ref, "err_vs_oracle"))
    rng = np.random.default_rng(0)
    pick = np.sort(rng.choice(sel.shape[0], size=256, replace=False))
    psel = sel[pick]
    bf, _ = oracle.attention_ref(gen["q"][one], gen["k"][one], gen["v"][one], gen["seqlens"][one], causal=True,
                                 sel=psel)
    res.update(_errs(got[pick], bf, "err_vs_bf16"))
    res.update(_errs(ref[pick], bf, "oracle_err_vs_bf16"))
    res["err_bf16_rows"] = "256 random rows of the subset"
    if p.get("rot_sub") is not None:
        rqc, rqs = oracle.quantize_qk_hadamard(gen["q"][one])
        rkc, rks = oracle.quantize_qk_hadamard(gen["k"][one], gen["seqlens"][one])
        ro, _ = oracle.attention(rqc, rqs, rkc, rks, vc, vs, gen["seqlens"][one], causal=True, sel=psel)
        rgot = np.transpose(p["rot_sub"], (1, 0, 2)).reshape(-1, 128)[pick]
        res.update(_errs(rgot, ro, "hadamard_err_vs_oracle"))
        res.update(_errs(rgot, bf, "hadamard_err_vs_bf16"))
    return res


def cpu_small_prefill_leg(s):
    import oracle
    gen, wl = s["gen"], s["wl"]
    n, sec = 0, 0.0
    while sec < 1.0:
        t = time.perf_counter()
        oz = oracle.quantize_workload(gen)
        ref, _ = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], gen["seqlens"],
                                  causal=True)
        sec += time.perf_counter() - t
        n += 1
    res = {"cpu_value": s["flops"] * n / sec / 1e12, "cpu_unit": "TFLOPS", "cpu_cores": oracle.num_threads(),
           "cpu_kind": "oracle", "cpu_seconds": sec,
           "cpu_sample": f"whole workload (quantize Q, K, V + attention), {n} repetitions"}
    res.update(_errs(s["out"], ref, "err_vs_oracle"))
    bf, _ = oracle.attention_ref(gen["q"], gen["k"], gen["v"], gen["seqlens"], causal=True)
    res.update(_errs(s["out"], bf, "err_vs_bf16"))
    res.update(_errs(ref, bf, "oracle_err_vs_bf16"))
    return res


def run_reference(args, world, rank):
    """--impl reference: the CPU oracle, as it stands, on the headline decode workload.

    One step is a bounded sample of the workload: one batch entry (its 8 KV
    heads, 8192 keys, 4 query rows each), MXFP4 query quantize + fp64 attention,
    the entry's cache quantized outside the timing (as on the GPU); when K + W
    such steps would take more than about three minutes, a step is one (b, h_kv)
    unit instead."""
    if rank != 0:
        return 0
    import oracle
    import synth
    wl = synth.WORKLOADS[DECODE_WORKLOAD]
    gen = wl.generate()
    cache = {}

    def entry(b):
        if b not in cache:
            kc, ks = oracle.quantize_qk(gen["k"][b:b + 1])
            vc, vs = oracle.quantize_v(gen["v"][b:b + 1], gen["seqlens"][b:b + 1])
            cache[b] = (kc, ks, vc, vs)
        return cache[b]

    def sub(arrs, h):
        kc, ks, vc, vs = arrs
        s = slice(h, h + 1)
        return kc[:, s], ks[:, s], vc[:, s], vs[:, s]

    G = wl.G
    mode = {"unit": False}

    def step(i):
        b = i % wl.B
        kc, ks, vc, vs = entry(b)
        if mode["unit"]:
            h = (i // wl.B) % wl.Hkv
            kc, ks, vc, vs = sub((kc, ks, vc, vs), h)
            qc, qs = oracle.quantize_qk(gen["q"][b:b + 1, :, h * G:(h + 1) * G])
        else:
            qc, qs = oracle.quantize_qk(gen["q"][b:b + 1])
        oracle.attention(qc, qs, kc, ks, vc, vs, gen["seqlens"][b:b + 1], causal=True)

    steps, warmup = max(1, args.steps), max(0, args.warmup)
    entry(0)
    t = time.perf_counter()
    step(0)
    one = time.perf_counter() - t
    if (steps + warmup) * one > 180.0:
        mode["unit"] = True
    step_bytes = (wl.Lk if mode["unit"] else wl.Hkv * wl.Lk) * KV_BYTES_PER_TOKEN_HEAD
    for i in range(warmup):
        step(i)
    for i in range(steps):
        entry(i % wl.B)   # the cache is quantized outside the timing
    t = time.perf_counter()
    for i in range(steps):
        step(i)
    sec = time.perf_counter() - t
    value = step_bytes * steps / sec / 1e9
    sample = ("one (b, h_kv) unit per step: 8192 keys, 4 query rows" if mode["unit"]
              else "one batch entry per step (of 32): 8 KV heads x 8192 keys, 4 query rows each")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": sec / steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------- main

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
    hbm_gbs, bf16_tf, peak_src = load_peaks()
    hadamard = not args.no_hadamard

    if args.quantize_only:
        if rank == 0:
            import synth
            gen = synth.WORKLOADS[PREFILL_WORKLOAD].generate()
            print(json.dumps({"quantize": run_quantize_kernels(hbm_gbs, gen, reps=3)}), flush=True)
        return 0
    if args.no_decode:
        if rank == 0:
            p = run_prefill(args, False)
            p["steps"] = args.prefill_steps
            print(json.dumps({"prefill": prefill_object(p, run_mma_peaks())}), flush=True)
        return 0

    d = run_decode(args, world, rank)
    wl = d["wl"]
    steps = args.steps
    value = aggregate_gbs(d["kv_bytes"], steps, world, d["elapsed_ms"])
    ms_per_step = d["elapsed_ms"] / steps
    achieved = d["kv_bytes"] / (d["attn_avg_ms"] * 1e-3) / 1e9
    e2e_value = aggregate_gbs(d["kv_bytes"], d["e2e_steps"], world, d["e2e_ms"])
    traffic = NCU_TRAFFIC.get(args.decode_workload)

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
        "config": headline_config(world) if args.decode_workload == DECODE_WORKLOAD else
        {"workload": args.decode_workload},
        "kv_splits": d["splits"],
        "tokens_per_s": wl.B * wl.Sq * steps * world / (d["elapsed_ms"] * 1e-3),
        "roofline": {
            "bound": "hbm", "kernel": decode_kernel_name(wl.G * wl.Sq),
            "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s", "frac": achieved / hbm_gbs,
            "frac_of_spec_8tbs": achieved / SPEC_HBM_GBS,
            "peak_source": f"{peak_src} hbm_gbs (burst copy)",
            "traffic": None if traffic is None else traffic[0],
            "traffic_source": None if traffic is None else traffic[1],
            "algorithmic_bytes_per_launch": d["kv_bytes"], "avg_launch_ms": d["attn_avg_ms"],
            "launch_timing": d["attn_timing"],
        },
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": d["h2d"], "d2h_bytes_per_step": d["d2h"],
                "steps": d["e2e_steps"],
                "how": "qk4v8_attention_decode_bf16 through the Python API; each step uploads its query from pinned "
                       "host memory and downloads its output, on two copy streams overlapping the next and previous "
                       "steps' kernels (double-buffered device buffers); the K steps replay as one CUDA graph"},
        "gpu_launches": d["launches_per_step"] * steps,
        "clocks": d["clocks"],
    }

    extra = {}
    v4 = {}
    draft = None
    if world == 1 and not args.no_extra_decode:
        for key, name in (("decode_long", LONG_WORKLOAD), ("verify", VERIFY_WORKLOAD)):
            extra[key] = run_decode_workload(name, args.extra_steps, min(args.warmup, 5), hbm_gbs,
                                             hadamard and key == "verify")
            line[key] = extra[key]["res"]
        # QK4V4, the article's comparison point, on the three decode workloads.
        for key, name, g in (("decode", DECODE_WORKLOAD, d["gen"]), ("decode_long", LONG_WORKLOAD,
                                                                        extra["decode_long"]["gen"]),
                             ("verify", VERIFY_WORKLOAD, extra["verify"]["gen"])):
            v4[key] = run_decode_v4(name, g, args.extra_steps, hbm_gbs)
        line["qk4v4"] = {"what": "V in MXFP4 (QK4V4) instead of MXFP8, same step, swap-AB kernel",
                         "decode_ms": v4["decode"]["ms"], "decode_gbs": v4["decode"]["gbs"],
                         "decode_speedup_vs_qk4v8": ms_per_step / v4["decode"]["ms"],
                         "decode_long_ms": v4["decode_long"]["ms"], "decode_long_gbs": v4["decode_long"]["gbs"],
                         "decode_long_speedup_vs_qk4v8": extra["decode_long"]["res"]["ms_per_step"] /
                         v4["decode_long"]["ms"],
                         "verify_ms": v4["verify"]["ms"], "verify_gbs": v4["verify"]["gbs"],
                         "verify_speedup_vs_qk4v8": extra["verify"]["res"]["ms_per_step"] / v4["verify"]["ms"],
                         "bytes_per_token_head": KV4_BYTES_PER_TOKEN_HEAD}
        line["paged"] = run_paged(d["gen"], args.extra_steps, hbm_gbs)
        draft = run_draft_block(extra["verify"]["gen"], hbm_gbs)
        line["draft_block"] = draft["res"]
    pre = small = None
    if world == 1 and not args.no_prefill:
        peaks = run_mma_peaks()
        line["mma_peaks"] = {**{k: v for k, v in peaks.items()}, "unit": "TFLOPS",
                             "how": "one CTA per SM issuing one tcgen05.mma shape from shared memory, CUDA events"}
        pre = run_prefill(args, hadamard)
        pre["steps"] = args.prefill_steps
        line["prefill"] = prefill_object(pre, peaks)
        small = run_prefill_small()
        line["prefill_small"] = small["res"]
        line["quantize"] = run_quantize_kernels(hbm_gbs, pre["gen"])

    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        head = cpu_decode_leg(d["gen"], wl, d["out"], None if d["rot"] is None else d["rot"][0],
                              v4["decode"]["out"] if "decode" in v4 else None)
        line["cpu_baseline"] = {"value": head["cpu_value"], "unit": "GB/s", "cores": head["cpu_cores"],
                                "kind": "oracle", "sample": head["cpu_sample"]}
        line["context_error"] = {k: v for k, v in head.items() if "err" in k}
        line["context_error"]["note"] = ("err_vs_oracle: GPU vs the fp64 QK4V8 oracle (bar: max 3e-2, mean 3e-3); "
                                         "err_vs_bf16: GPU vs fp64 attention over the unquantized bf16 inputs "
                                         "(context, no bar); hadamard_*: Q and K quantized after rotation; "
                                         "qk4v4_*: V in MXFP4 (against the QK4V4 oracle)")
        if d["rot"] is not None:
            line["context_error"]["hadamard_ms_per_step"] = d["rot"][1]
        for key, x in extra.items():
            x["res"].update(cpu_decode_leg(x["gen"], x["wl"], x["out"], x["rot"],
                                           v4[key]["out"] if key in v4 else None))
        if draft is not None:
            line["draft_block"].update(cpu_draft_block_leg(extra["verify"]["gen"], extra["verify"]["wl"],
                                                           draft["out"], draft["window"]))
        if pre is not None:
            line["prefill"].update(cpu_prefill_leg(pre))
        if small is not None:
            line["prefill_small"].update(cpu_small_prefill_leg(small))

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
