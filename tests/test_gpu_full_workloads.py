"""Parity at the full workload sizes, in the launch configuration bench.py times.

The GPU runs the whole workload exactly as the benchmark does: the decode
workloads through qk4v8_attention_decode_bf16 with the library's default split
count over the pre-quantized cache, the prefill workload through
qk4v8_quantize followed by causal qk4v8_attention_prefill. The fp64 oracle
then quantizes the sampled batch entries itself, from the same bf16 inputs,
and computes the sampled output rows one by one. Tolerance as everywhere:
max-abs 3e-2 and mean-abs 3e-3 on the attention output; 1e-2 on the
log-sum-exp.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import oracle
import synth
from gpu_util import MAX_ABS_TOL, MEAN_ABS_TOL, to_dev

pytestmark = pytest.mark.gpu


def oracle_rows(gen, b, rows, causal):
    """Oracle output rows (h_q, i) of batch entry b, quantizing that entry itself."""
    one = slice(b, b + 1)
    qc, qs = oracle.quantize_qk(gen["q"][one])
    kc, ks = oracle.quantize_qk(gen["k"][one])
    vc, vs = oracle.quantize_v(gen["v"][one], gen["seqlens"][one])
    sel = np.array([(0, h, i) for h, i in rows], dtype=np.int32)
    return oracle.attention(qc, qs, kc, ks, vc, vs, gen["seqlens"][one], causal=causal, sel=sel)


def check(got, ref, got_lse, ref_lse, what):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    d = np.abs(got - ref)
    assert d.max() <= MAX_ABS_TOL and d.mean() <= MEAN_ABS_TOL, f"{what}: max-abs {d.max():.4g} mean-abs {d.mean():.4g}"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got_lse), fin), what
    assert np.abs(got_lse[fin] - ref_lse[fin]).max() < 1e-2, what


@pytest.mark.timeout(600)
@pytest.mark.parametrize("name", ["decode_gqa_b32_hq32_hkv8_l8192", "decode_long_b8_hq64_hkv8_l64k_128k",
                                  "verify_b64_nq8_hq64_hkv8_l16384"])
def test_decode_workload_full_size(name):
    wl = synth.WORKLOADS[name]
    gen = wl.generate()
    lens = gen["seqlens"]
    sl = torch.from_numpy(lens).cuda()
    cap = qk.round_cap(wl.Lk)
    kp = qk.quantize_qk(to_dev(gen["k"]), cap=cap, seqlens=sl)
    vp = qk.quantize_v(to_dev(gen["v"]), cap=cap, seqlens=sl)
    q = to_dev(gen["q"])
    max_len = int(lens.max())
    # The split count bench.py times: the plan from the host-side lengths.
    splits = qk.decode_plan_splits(wl.B, wl.Hq, wl.Hkv, wl.Sq, lens)
    out, lse = qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=max_len, num_splits=splits, return_lse=True)
    torch.cuda.synchronize()
    out = out.float().cpu().numpy()   # [B, nq, Hq, d]
    lse = lse.cpu().numpy()           # [B, Hq, nq]
    del kp, vp
    for b in sorted({0, wl.B // 2, wl.B - 1}):
        rows = [(h, t) for h in range(wl.Hq) for t in range(wl.Sq)]
        ref, rlse = oracle_rows(gen, b, rows, causal=True)
        got = np.stack([out[b, t, h] for h, t in rows]).astype(np.float64)
        glse = np.array([lse[b, h, t] for h, t in rows], dtype=np.float64)
        check(got, ref, glse, rlse, f"{name} b={b} (splits {splits})")


@pytest.mark.timeout(600)
def test_prefill_workload_full_size():
    name = "prefill_gqa_b4_hq32_hkv8_s8192"
    wl = synth.WORKLOADS[name]
    gen = wl.generate()
    q, k, v = to_dev(gen["q"]), to_dev(gen["k"]), to_dev(gen["v"])
    qp, kp, vp = qk.quantize(q, k, v)
    out, lse = qk.attention_prefill(qp, kp, vp, causal=True, return_lse=True)
    torch.cuda.synchronize()
    out = out.float().cpu().numpy()   # [B, S, Hq, d]
    lse = lse.cpu().numpy()           # [B, Hq, S]
    del q, k, v, qp, kp, vp
    rng = np.random.default_rng(7)
    S = wl.Sq
    for b in (0, wl.B - 1):
        # Random rows, plus the first and last rows and both sides of a tile edge.
        rows = [(int(h), int(i)) for h, i in zip(rng.integers(0, wl.Hq, 96), rng.integers(0, S, 96))]
        rows += [(0, 0), (wl.Hq - 1, S - 1), (3, 127), (3, 128), (17, S - 128), (17, S - 129)]
        ref, rlse = oracle_rows(gen, b, rows, causal=True)
        got = np.stack([out[b, i, h] for h, i in rows]).astype(np.float64)
        glse = np.array([lse[b, h, i] for h, i in rows], dtype=np.float64)
        check(got, ref, glse, rlse, f"{name} b={b}")


@pytest.mark.timeout(900)
@pytest.mark.parametrize("name", ["decode_gqa_b32_hq32_hkv8_l8192", "decode_long_b8_hq64_hkv8_l64k_128k",
                                  "verify_b64_nq8_hq64_hkv8_l16384"])
def test_qk4v4_workload_full_size(name):
    """QK4V4 (V in MXFP4) at full size, as bench.py runs it: bf16 queries, the planned splits."""
    wl = synth.WORKLOADS[name]
    gen = wl.generate()
    lens = gen["seqlens"]
    sl = torch.from_numpy(lens).cuda()
    cap = qk.round_cap(wl.Lk)
    kp = qk.quantize_qk(to_dev(gen["k"]), cap=cap, seqlens=sl)
    vp = qk.quantize_v4(to_dev(gen["v"]), cap=cap, seqlens=sl)
    max_len = int(lens.max())
    splits = qk.decode_plan_splits(wl.B, wl.Hq, wl.Hkv, wl.Sq, lens)
    out, lse = qk.attention_decode_bf16(to_dev(gen["q"]), kp, vp, sl, max_seqlen=max_len, num_splits=splits,
                                        return_lse=True)
    torch.cuda.synchronize()
    out = out.float().cpu().numpy()
    lse = lse.cpu().numpy()
    del kp, vp
    for b in sorted({0, wl.B - 1}):
        one = slice(b, b + 1)
        sub = dict(q=gen["q"][one], k=gen["k"][one], v=gen["v"][one], seqlens=lens[one])
        oz = oracle.quantize_workload(sub, v_fmt=oracle.E2M1)
        rows = [(h, t) for h in range(wl.Hq) for t in range(wl.Sq)]
        sel = np.array([(0, h, t) for h, t in rows], dtype=np.int32)
        ref, rlse = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], lens[one],
                                     causal=True, sel=sel, v_fmt=oracle.E2M1)
        got = np.stack([out[b, t, h] for h, t in rows]).astype(np.float64)
        glse = np.array([lse[b, h, t] for h, t in rows], dtype=np.float64)
        check(got, ref, glse, rlse, f"QK4V4 {name} b={b}")


@pytest.mark.timeout(900)
def test_draft_block_window_full_size():
    """The draft-block window (1024 keys before the 8-token block, non-causal) on the
    speculative-verify workload's full cache, as bench.py runs it."""
    name = "verify_b64_nq8_hq64_hkv8_l16384"
    wl = synth.WORKLOADS[name]
    gen = wl.generate()
    lens = gen["seqlens"]
    sl = torch.from_numpy(lens).cuda()
    cap = qk.round_cap(wl.Lk)
    kp = qk.quantize_qk(to_dev(gen["k"]), cap=cap, seqlens=sl)
    vp = qk.quantize_v(to_dev(gen["v"]), cap=cap, seqlens=sl)
    out, lse = qk.attention_decode_bf16(to_dev(gen["q"]), kp, vp, sl, max_seqlen=wl.Lk, causal_in_block=False,
                                        window=1024, return_lse=True)
    torch.cuda.synchronize()
    out = out.float().cpu().numpy()
    lse = lse.cpu().numpy()
    del kp, vp
    for b in (0, wl.B // 2, wl.B - 1):
        one = slice(b, b + 1)
        sub = dict(q=gen["q"][one], k=gen["k"][one], v=gen["v"][one], seqlens=lens[one])
        oz = oracle.quantize_workload(sub)
        rows = [(h, t) for h in range(wl.Hq) for t in range(wl.Sq)]
        sel = np.array([(0, h, t) for h, t in rows], dtype=np.int32)
        ref, rlse = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], lens[one],
                                     causal=False, sel=sel, window=1024)
        got = np.stack([out[b, t, h] for h, t in rows]).astype(np.float64)
        glse = np.array([lse[b, h, t] for h, t in rows], dtype=np.float64)
        check(got, ref, glse, rlse, f"draft block b={b}")


@pytest.mark.timeout(900)
def test_paged_headline_full_size():
    """The headline decode workload over a paged cache built by appending the
    whole prompt (then 3 decode tokens) into pages in random order: the pages
    must hold the oracle's bytes for the appended tokens, and the decode must
    match the oracle."""
    wl = synth.WORKLOADS["decode_gqa_b32_hq32_hkv8_l8192"]
    gen = wl.generate()
    B, L = wl.B, wl.Lk
    prompt = L - 3
    max_pages = L // 128 + 1
    num_pages = B * max_pages
    perm = np.random.default_rng(1).permutation(num_pages).astype(np.int32).reshape(B, max_pages)
    cache = qk.paged_kv(B, wl.Hkv, num_pages, torch.from_numpy(perm))
    k, v = to_dev(gen["k"]), to_dev(gen["v"])
    qk.kv_append(cache, k[:, :prompt], v[:, :prompt])
    for t in range(prompt, L):
        qk.kv_append(cache, k[:, t:t + 1], v[:, t:t + 1])
    out = qk.attention_decode_bf16_paged(to_dev(gen["q"]), cache, max_seqlen=L)
    torch.cuda.synchronize()
    assert cache.seqlens.cpu().tolist() == [L] * B
    out = out.float().cpu().numpy()
    for b in (0, B - 1):
        one = slice(b, b + 1)
        sub = dict(q=gen["q"][one], k=gen["k"][one], v=gen["v"][one], seqlens=gen["seqlens"][one])
        oz = oracle.quantize_workload(sub)
        ref, _ = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], sub["seqlens"],
                                  causal=True)
        d = np.abs(out[b] - ref[0])
        assert d.max() <= MAX_ABS_TOL and d.mean() <= MEAN_ABS_TOL, (b, d.max(), d.mean())
