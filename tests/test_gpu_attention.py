"""QK4V8 attention on the GPU against the fp64 CPU oracle.

Bar: attention output within max-abs 3e-2 and mean-abs 3e-3 of the oracle for
unit-variance inputs. The GPU quantizes with the library's own kernels, and
test_gpu_quantize checks that step bit-exactly, so both sides attend over
identical MX tensors.
"""
import math

import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import oracle
import synth
from bit_quantized_attention_qk4v8_b200 import _lib
from gpu_util import assert_close, err_stats, oracle_attention_from, packed_to_logical, quantize_on_gpu, to_dev
from layouts import fill_v_bytes, qk_scales_logical, unpack_e2m1

pytestmark = pytest.mark.gpu

E2M1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def f32_to_bf16_bits(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def make_gen(B, Sq, Lk, Hq, Hkv, seed, lens=None, q_scale=1.0, k_out=0, mult=16.0):
    wl = synth.Workload("t", "decode", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Lk=Lk, seed=seed, k_outliers=k_out,
                        q_outliers=k_out > 0, outlier_mult=mult)
    gen = wl.generate()
    if lens is not None:
        gen["seqlens"] = np.array(lens, dtype=np.int32)
        for b, L in enumerate(lens):
            gen["k"][b, L:] = 0
            gen["v"][b, L:] = 0
    if q_scale != 1.0:
        q = (gen["q"].astype(np.uint32) << 16).view(np.float32) * np.float32(q_scale)
        gen["q"] = f32_to_bf16_bits(q)
    return gen


def run_prefill(gen, causal, scale=None):
    qp, kp, vp, sl = quantize_on_gpu(gen)
    out, lse = qk.attention_prefill(qp, kp, vp, seqlens_k=sl, causal=causal, softmax_scale=scale, return_lse=True)
    torch.cuda.synchronize()
    return out, lse, (qp, kp, vp)


def run_decode(gen, causal=True, splits=0, scale=None):
    qp, kp, vp, sl = quantize_on_gpu(gen)
    out, lse = qk.attention_decode(qp, kp, vp, sl, max_seqlen=int(gen["seqlens"].max()), causal_in_block=causal,
                                   num_splits=splits, softmax_scale=scale, return_lse=True)
    torch.cuda.synchronize()
    return out, lse, (qp, kp, vp)


def test_scores_tile_matches_dequantized_dot_products():
    """The block-scaled FP4 MMA alone: raw S = Q K^T of one 128x128 tile."""
    gen = make_gen(1, 128, 128, 1, 1, seed=21, k_out=4)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    dump = torch.zeros((128, 128), dtype=torch.float32, device="cuda")
    _lib.lib().qk4v8_test_set_dump_scores(dump.data_ptr())
    try:
        qk.attention_prefill(qp, kp, vp, seqlens_k=sl, causal=False)
        torch.cuda.synchronize()
    finally:
        _lib.lib().qk4v8_test_set_dump_scores(None)
    lz = packed_to_logical(qp, kp, vp, 128, 128)

    def deq(c, s):
        v = E2M1[c & 7] * np.where(c & 8, -1.0, 1.0)
        return v * np.exp2(np.repeat(s.astype(np.float64) - 127, 32, axis=-1))

    qd = deq(lz["qc"][0, 0], lz["qs"][0, 0])
    kd = deq(lz["kc"][0, 0], lz["ks"][0, 0])
    ref = qd @ kd.T
    got = dump.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


@pytest.mark.parametrize("B,S,Hq,Hkv,causal", [
    (1, 256, 2, 2, True),      # the small causal prefill workload's shape
    (1, 200, 2, 1, True),      # ragged query and key tiles, GQA 2
    (2, 128, 4, 1, False),     # non-causal, GQA 4
    (1, 384, 8, 2, True),      # several key tiles
    (1, 1, 1, 1, True),        # a single token
    (4, 256, 64, 8, True),     # 512 units: several per CTA, Q buffers and the K and V rings reused across units
])
def test_prefill_parity(B, S, Hq, Hkv, causal):
    gen = make_gen(B, S, S, Hq, Hkv, seed=S + Hq)
    out, lse, _ = run_prefill(gen, causal)
    (ref, rlse), _ = oracle_attention_from(gen, causal)
    assert_close(out, ref, f"prefill B{B} S{S} Hq{Hq} Hkv{Hkv} causal{causal}")
    l = lse.cpu().numpy().transpose(0, 2, 1)
    assert np.abs(l - rlse).max() < 1e-2


def test_prefill_workload_small_full():
    wl = synth.WORKLOADS["prefill_b1_h2_s256"]
    gen = wl.generate()
    out, _, _ = run_prefill(gen, True)
    (ref, _), _ = oracle_attention_from(gen, True)
    assert_close(out, ref, wl.name)


def test_prefill_varlen_keys_and_offsets():
    """Varlen KV shorter and longer than the query block; causal bottom-right offsets."""
    gen = make_gen(3, 64, 300, 4, 2, seed=5, lens=[300, 64, 37])
    for causal in (True, False):
        out, _, _ = run_prefill(gen, causal)
        (ref, _), _ = oracle_attention_from(gen, causal)
        assert_close(out, ref, f"varlen causal={causal}")


def test_prefill_empty_rows():
    """Keys fewer than queries under causal masking: early rows see no key at all."""
    gen = make_gen(2, 100, 100, 2, 2, seed=8, lens=[40, 0])
    out, lse, _ = run_prefill(gen, True)
    (ref, rlse), _ = oracle_attention_from(gen, True)
    assert_close(out, ref, "empty rows")
    l = lse.cpu().numpy().transpose(0, 2, 1)
    assert np.array_equal(np.isinf(l), np.isinf(rlse))
    assert (out[1].float().abs().max() == 0)


def test_prefill_softmax_scale_and_peaked_scores():
    gen = make_gen(1, 256, 256, 2, 1, seed=13, q_scale=3.0, k_out=2, mult=20.0)
    out, _, _ = run_prefill(gen, True, scale=0.2)
    (ref, _), _ = oracle_attention_from(gen, True, scale=0.2)
    assert_close(out, ref, "custom scale, peaked")


@pytest.mark.parametrize("B,nq,L,Hq,Hkv,splits,lens", [
    (2, 1, 1000, 8, 2, 0, None),
    (2, 1, 4096, 32, 8, 3, None),
    (3, 8, 700, 16, 2, 2, None),
    (4, 1, 2000, 8, 8, 5, [2000, 1, 33, 129]),
    (2, 8, 1024, 64, 8, 1, [1024, 500]),
    (2, 4, 300, 4, 1, 7, [300, 7]),
    (1, 8, 600, 16, 1, 2, None),       # G*nq = 128 rows: the 128-row kernel's decode path
    (2, 3, 900, 12, 4, 3, [900, 400]), # odd row count (G*nq = 9)
    (2, 2, 1500, 16, 4, 2, None),      # G*nq = 8: the 8-row instance
    (2, 1, 3000, 64, 8, 1, [3000, 2999]),  # GQA 8, one token: 8 rows, one split (direct output)
    (2, 5, 700, 5, 5, 2, [700, 64]),   # G*nq = 5
    (2, 4, 800, 32, 4, 2, [800, 511]),  # G*nq = 32: the 32-row instance
    (2, 8, 1100, 24, 4, 0, [1100, 513]),  # G*nq = 48: the GQA decode kernel, odd tile counts
    (1, 3, 900, 11, 1, 2, None),          # G*nq = 33: the GQA decode kernel's smallest group
    (3, 8, 1000, 64, 8, 3, [1000, 129, 1]),  # 64 rows, splits of 3 tiles, a one-tile and a one-key sequence
    (2, 4, 2300, 16, 1, 1, [2300, 2001]),  # 64 rows from 16 heads x 4 tokens, direct output
])
def test_decode_parity(B, nq, L, Hq, Hkv, splits, lens):
    gen = make_gen(B, nq, L, Hq, Hkv, seed=L + nq, lens=lens, k_out=4)
    out, lse, _ = run_decode(gen, True, splits)
    (ref, rlse), _ = oracle_attention_from(gen, True)
    assert_close(out, ref, f"decode B{B} nq{nq} L{L} Hq{Hq} Hkv{Hkv} splits{splits}")
    l = lse.cpu().numpy().transpose(0, 2, 1)
    fin = np.isfinite(rlse)
    assert np.abs(l[fin] - rlse[fin]).max() < 1e-2


def test_decode_edge_lengths():
    lens = [1, 31, 32, 33, 127, 128, 129, 255]
    gen = make_gen(len(lens), 1, 256, 8, 2, seed=77, lens=lens, k_out=4)
    for splits in (1, 2):
        out, _, _ = run_decode(gen, True, splits)
        (ref, _), _ = oracle_attention_from(gen, True)
        assert_close(out, ref, f"edge lengths splits={splits}")


def test_decode_zero_length_sequence():
    gen = make_gen(2, 2, 256, 4, 2, seed=3, lens=[256, 0])
    out, lse, _ = run_decode(gen, True, 2)
    assert out[1].float().abs().max().item() == 0
    assert torch.isinf(lse[1]).all()
    (ref, _), _ = oracle_attention_from(gen, True)
    assert_close(out, ref, "zero-length")


def test_decode_poisoned_padding_does_not_leak():
    """Cache bytes past each sequence's length are overwritten with NaN patterns."""
    gen = make_gen(2, 1, 512, 8, 2, seed=4, lens=[300, 45], k_out=4)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    clean = qk.attention_decode(qp, kp, vp, sl, max_seqlen=300, num_splits=2)
    for b, L in enumerate([300, 45]):
        fill_v_bytes(vp.codes, b, L, 0xFF)    # E4M3 NaN
        kp.codes[b, :, L:] = 0xFF
        blk0 = L // 128
        # scale atoms of blocks fully past L, and the groups past L inside block blk0
        vp.scales[b, :, blk0 + 1:] = 0xFF
        kp.scales[b, :, blk0 + 1:] = 0xFF
        jv = L - blk0 * 128
        idx = torch.tensor([(c % 32) * 16 + (c // 32) * 4 + g for c in range(128) for g in range((jv + 31) // 32, 4)],
                           dtype=torch.long, device="cuda")
        if idx.numel():
            vp.scales[b, :, blk0, idx] = 0xFF
        tidx = torch.tensor([(t % 32) * 16 + (t // 32) * 4 + g for t in range(jv, 128) for g in range(4)],
                            dtype=torch.long, device="cuda")
        kp.scales[b, :, blk0, tidx] = 0xFF
    dirty = qk.attention_decode(qp, kp, vp, sl, max_seqlen=300, num_splits=2)
    torch.cuda.synchronize()
    assert torch.isfinite(dirty.float()).all()
    assert torch.equal(clean, dirty)


def _poison_padding(kp, vp, lens):
    """Overwrite every cache byte past each sequence's length with NaN patterns:
    codes, whole scale atoms past the last block, and the scale entries of the
    padding rows and groups inside the last block."""
    for b, L in enumerate(lens):
        fill_v_bytes(vp.codes, b, L, 0xFF)    # E4M3 NaN
        kp.codes[b, :, L:] = 0xFF
        blk0 = L // 128
        vp.scales[b, :, blk0 + 1:] = 0xFF
        kp.scales[b, :, blk0 + 1:] = 0xFF
        jv = L - blk0 * 128
        if blk0 >= vp.scales.shape[2]:
            continue
        if jv == 0:   # block blk0 starts at L: all of it is padding
            vp.scales[b, :, blk0] = 0xFF
            kp.scales[b, :, blk0] = 0xFF
            continue
        idx = torch.tensor([(c % 32) * 16 + (c // 32) * 4 + g for c in range(128) for g in range((jv + 31) // 32, 4)],
                           dtype=torch.long, device="cuda")
        if idx.numel():
            vp.scales[b, :, blk0, idx] = 0xFF
        tidx = torch.tensor([(t % 32) * 16 + (t // 32) * 4 + g for t in range(jv, 128) for g in range(4)],
                            dtype=torch.long, device="cuda")
        kp.scales[b, :, blk0, tidx] = 0xFF


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_poisoned_padding_does_not_leak(causal):
    """Prefill over a cache whose bytes past each length are NaN patterns: the
    output must equal the one over clean (zero) padding, bit for bit."""
    lens = [300, 45, 256]
    gen = make_gen(3, 64, 512, 8, 2, seed=14, lens=lens, k_out=2)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    clean = qk.attention_prefill(qp, kp, vp, seqlens_k=sl, causal=causal)
    torch.cuda.synchronize()
    clean = clean.clone()
    _poison_padding(kp, vp, lens)
    dirty = qk.attention_prefill(qp, kp, vp, seqlens_k=sl, causal=causal)
    torch.cuda.synchronize()
    assert torch.isfinite(dirty.float()).all()
    assert torch.equal(clean, dirty)
    (ref, _), _ = oracle_attention_from(gen, causal)
    assert_close(dirty, ref, f"poisoned prefill causal={causal}")


@pytest.mark.parametrize("Hq,Hkv,nq,splits", [(64, 8, 8, 3), (16, 1, 8, 2)])
def test_decode_poisoned_padding_larger_groups(Hq, Hkv, nq, splits):
    """The GQA decode kernel (64 rows) and the 128-row kernel over NaN padding."""
    lens = [300, 45, 129]
    gen = make_gen(3, nq, 512, Hq, Hkv, seed=15, lens=lens, k_out=4)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    clean = qk.attention_decode(qp, kp, vp, sl, max_seqlen=300, num_splits=splits)
    torch.cuda.synchronize()
    clean = clean.clone()
    _poison_padding(kp, vp, lens)
    dirty = qk.attention_decode(qp, kp, vp, sl, max_seqlen=300, num_splits=splits)
    torch.cuda.synchronize()
    assert torch.isfinite(dirty.float()).all()
    assert torch.equal(clean, dirty)


def test_deterministic():
    gen = make_gen(2, 8, 1500, 16, 2, seed=9, k_out=4)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    a = qk.attention_decode(qp, kp, vp, sl, max_seqlen=1500, num_splits=3)
    b = qk.attention_decode(qp, kp, vp, sl, max_seqlen=1500, num_splits=3)
    gp = make_gen(1, 300, 300, 4, 2, seed=2)
    pq, pk, pv, psl = quantize_on_gpu(gp)
    c = qk.attention_prefill(pq, pk, pv, seqlens_k=psl)
    d = qk.attention_prefill(pq, pk, pv, seqlens_k=psl)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(c, d)


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,lens", [
    (2, 100, 300, 4, 2, [300, 150]),
    (5, 1, 1000, 8, 2, [1000, 1, 0, 999, 512]),   # one launch: Q, K and V CTAs of five entries
])
def test_quantize_entry_point_matches_separate_calls(B, Sq, Sk, Hq, Hkv, lens):
    gen = make_gen(B, Sq, Sk, Hq, Hkv, seed=12, lens=lens)
    q, k, v = to_dev(gen["q"]), to_dev(gen["k"]), to_dev(gen["v"])
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    qp, kp, vp = qk.quantize(q, k, v, seqlens_k=sl)
    qp2, kp2, vp2, _ = quantize_on_gpu(gen)
    torch.cuda.synchronize()
    for a, b in ((qp, qp2), (kp, kp2), (vp, vp2)):
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)


def dequantized_scores(qp, kp, Sq, Lk):
    """fp64 S = Q K^T (no softmax scale) of the dequantized packed tensors, [B, Hq, Sq, Lk] per KV group."""
    qc = unpack_e2m1(qp.codes.cpu().numpy()[:, :, :Sq])
    qs = qk_scales_logical(qp.scales.cpu().numpy(), Sq)
    kc = unpack_e2m1(kp.codes.cpu().numpy()[:, :, :Lk])
    ks = qk_scales_logical(kp.scales.cpu().numpy(), Lk)

    def deq(c, s):
        v = E2M1[c & 7] * np.where(c & 8, -1.0, 1.0)
        return v * np.exp2(np.repeat(s.astype(np.float64) - 127, 32, axis=-1))

    qd, kd = deq(qc, qs), deq(kc, ks)
    G = qd.shape[1] // kd.shape[1]
    kd = np.repeat(kd, G, axis=1)
    return np.einsum("bhid,bhjd->bhij", qd, kd)


@pytest.mark.parametrize("B,S,Hq,Hkv,causal,lens", [
    (1, 384, 4, 2, True, None),
    (2, 200, 2, 1, False, [200, 77]),
    (2, 130, 2, 2, True, [130, 0]),
    # several units per CTA (512 units on at most 148 CTAs), of one and two key
    # tiles, so the two tile parities of a CTA drift apart across units
    (4, 256, 64, 8, True, None),
    (8, 256, 32, 8, False, [256, 1, 129, 128, 0, 77, 255, 3]),
])
def test_prefill_stage_qk_row_max(B, S, Hq, Hkv, causal, lens):
    """The QK^T-stage build: each row's largest allowed scaled score, exactly as the scores' max."""
    gen = make_gen(B, S, S, Hq, Hkv, seed=S + 3, lens=lens, k_out=2, mult=20.0)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    rm = qk.prefill_stage_qk(qp, kp, seqlens_k=sl, causal=causal)
    torch.cuda.synchronize()
    s = dequantized_scores(qp, kp, S, S)
    c = (1.0 / math.sqrt(128)) * math.log2(math.e)
    L = gen["seqlens"]
    ref = np.full((B, Hq, S), -np.inf)
    for b in range(B):
        for i in range(S):
            lim = L[b] if not causal else min(L[b], i + L[b] - S + 1)
            if lim > 0:
                ref[b, :, i] = s[b, :, i, :lim].max(axis=-1) * c
    got = rm.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin)
    # fp32 accumulation of exact FP4 products: relative error ~1e-6
    assert np.abs(got[fin] - ref[fin]).max() <= 1e-5 * max(1.0, np.abs(ref[fin]).max())


def test_prefill_o_rescale_path():
    """Later keys score far (>64 binades) above the first tile's row max, so O is rescaled mid-row."""
    gen = make_gen(1, 128, 512, 2, 1, seed=41)
    k = (gen["k"].astype(np.uint32) << 16).view(np.float32).copy()
    k[:, :128] *= np.float32(1e-3)      # the first key tile: near-zero scores
    gen["k"] = f32_to_bf16_bits(k)
    scale = 6.0                          # scores of the later tiles reach ~100 binades
    out, lse, _ = run_prefill(gen, False, scale=scale)
    (ref, rlse), _ = oracle_attention_from(gen, False, scale=scale)
    assert_close(out, ref, "prefill O rescale")
    l = lse.cpu().numpy().transpose(0, 2, 1)
    assert np.abs(l - rlse).max() < 1e-2 + 1e-5 * np.abs(rlse).max()


@pytest.mark.parametrize("B,nq,L,Hq,Hkv,splits", [
    (2, 8, 1500, 64, 8, 1),
    (2, 8, 1500, 40, 8, 2),
])
def test_gqa_decode_kernel_agrees_with_swap_ab_kernel(B, nq, L, Hq, Hkv, splits):
    """33..64 query rows per KV head: the GQA decode kernel and the swap-AB kernel
    (selected by a test hook) compute the same attention, each within the
    oracle's tolerance."""
    gen = make_gen(B, nq, L, Hq, Hkv, seed=L + Hq, k_out=4)
    (ref, rlse), _ = oracle_attention_from(gen, True)
    out_gqa, lse_gqa, _ = run_decode(gen, True, splits)
    _lib.lib().qk4v8_test_set_force_swap_ab(1)
    try:
        out_swap, lse_swap, _ = run_decode(gen, True, splits)
    finally:
        _lib.lib().qk4v8_test_set_force_swap_ab(0)
    assert_close(out_gqa, ref, "GQA decode kernel")
    assert_close(out_swap, ref, "swap-AB kernel")
    fin = np.isfinite(rlse)
    for lse in (lse_gqa, lse_swap):
        l = lse.cpu().numpy().transpose(0, 2, 1)
        assert np.abs(l[fin] - rlse[fin]).max() < 1e-2


def test_gqa_decode_o_rescale_path():
    """64 rows per KV head; later keys score far (>64 binades) above the first
    tile's row max, so the GQA decode kernel rescales O mid-row (both lanes of
    each row, agreed between the two threads that own them)."""
    gen = make_gen(1, 8, 1024, 16, 2, seed=43)
    k = (gen["k"].astype(np.uint32) << 16).view(np.float32).copy()
    k[:, :128] *= np.float32(1e-3)      # the first key tile: near-zero scores
    gen["k"] = f32_to_bf16_bits(k)
    scale = 6.0
    for splits in (1, 2):
        out, lse, _ = run_decode(gen, False, splits, scale=scale)
        (ref, rlse), _ = oracle_attention_from(gen, False, scale=scale)
        assert_close(out, ref, f"GQA decode O rescale, splits={splits}")
        l = lse.cpu().numpy().transpose(0, 2, 1)
        assert np.abs(l - rlse).max() < 1e-2 + 1e-5 * np.abs(rlse).max()


@pytest.mark.parametrize("B,nq,L,Hq,Hkv,splits,lens", [
    # 8 x 8 sequences of 32 tiles over one CTA per SM: each CTA's even share of
    # the 2048 tiles is 13 or 14, so sequences are cut into up to 4 pieces.
    (8, 8, 4096, 64, 8, 4, None),
    # Mixed lengths (empty, one key, a few tiles, long): whole sequences, pieces
    # spread over up to 17 CTAs, and empty sequences inside the tile list.
    (16, 8, 4096, 16, 2, 20, [4096, 0, 1, 129, 4096, 3000, 0, 255, 4000, 17, 2048, 4096, 1024, 0, 3500, 640]),
])
def test_gqa_decode_balanced_schedule(B, nq, L, Hq, Hkv, splits, lens):
    """GQA decode with the balanced schedule: key tiles of all sequences spread
    evenly over the CTAs, sequences cut at the CTA range boundaries merged by
    the follow-up launch. Checked against the oracle, and against a one-split
    run of the same kernel (each sequence whole in one CTA)."""
    gen = make_gen(B, nq, L, Hq, Hkv, seed=L + B + splits, lens=lens, k_out=4)
    (ref, rlse), _ = oracle_attention_from(gen, True)
    out, lse, _ = run_decode(gen, True, splits)
    one, one_lse, _ = run_decode(gen, True, 1)
    assert_close(out, ref, f"balanced GQA decode B{B} splits{splits}")
    assert_close(one, ref, f"one-split GQA decode B{B}")
    fin = np.isfinite(rlse)
    for got in (lse, one_lse):
        l = got.cpu().numpy().transpose(0, 2, 1)
        assert np.array_equal(np.isfinite(l), fin)
        assert np.abs(l[fin] - rlse[fin]).max() < 1e-2
    # The same call twice gives the same bits.
    again, _, _ = run_decode(gen, True, splits)
    assert torch.equal(out, again)
