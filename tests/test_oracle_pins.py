"""Pins for the CPU oracle, checked against things other than the oracle itself.

Each pin uses an independent formulation: the OCP MX element grids (golden
fixture), torch's own float8_e4m3fn decoding, brute-force nearest-grid search
in numpy, hand-worked rounding/scale tables, closed forms of softmax attention,
and a naive numpy attention written here from the definition. A mistake in the
oracle (a dropped scale term, a wrong tie rule, a wrong GQA head or causal
offset) changes at least one of these results.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "mx_formats.json")))
E2M1_MAG = np.array(GOLD["e2m1_magnitudes"], dtype=np.float64)
E4M3_ALL = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def f32_to_bf16_bits(x):
    """Round float32 to bf16 (nearest even) and return the bit pattern."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f64(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- element grids

def test_e2m1_grid_matches_standard_and_roundtrips():
    for code in range(16):
        v = oracle.decode(oracle.E2M1, code)
        mag = E2M1_MAG[code & 7]
        assert v == (-mag if code & 8 else mag)
        assert oracle.encode(oracle.E2M1, v) == code


def test_e4m3_grid_matches_torch_and_roundtrips():
    for code in range(256):
        v = oracle.decode(oracle.E4M3, code)
        if code in GOLD["e4m3_nan_codes"]:
            assert math.isnan(v)
            continue
        assert v == E4M3_ALL[code] or (v == 0 and E4M3_ALL[code] == 0)
        assert math.copysign(1, v) == math.copysign(1, E4M3_ALL[code])
        assert oracle.encode(oracle.E4M3, v) == code
    assert oracle.decode(oracle.E4M3, 0x7E) == GOLD["e4m3_max"]
    assert oracle.decode(oracle.E4M3, 0x08) == GOLD["e4m3_min_normal"]
    assert oracle.decode(oracle.E4M3, 0x01) == GOLD["e4m3_min_subnormal"]


@pytest.mark.parametrize("fmt,key", [(oracle.E2M1, "worked_rne_e2m1"), (oracle.E4M3, "worked_rne_e4m3")])
def test_rne_worked_table(fmt, key):
    for y, expect in GOLD[key]["cases"]:
        code = oracle.encode(fmt, y)
        v = oracle.decode(fmt, code)
        assert v == expect, (y, v, expect)
        assert math.copysign(1, v) == math.copysign(1, y)  # sign of zero follows the input


@pytest.mark.parametrize("fmt,key", [(oracle.E2M1, "e2m1"), (oracle.E4M3, "e4m3")])
def test_scale_worked_values(fmt, key):
    for amax, byte in GOLD["worked_scales"][key]:
        x = np.zeros((1, 32), dtype=np.uint16)
        x[0, 5] = f32_to_bf16_bits(np.float32(amax))
        x[0, 9] = f32_to_bf16_bits(np.float32(-amax / 3))
        _, s = oracle.quantize_rows(x, fmt)
        assert int(s[0, 0]) == byte, (amax, int(s[0, 0]), byte)


# ------------------------------------------------- exhaustive brute-force encoder

def _grid(fmt):
    if fmt == oracle.E2M1:
        return E2M1_MAG, 0x8
    mags = E4M3_ALL[:127].copy()  # magnitude codes 0..126 (127 is NaN)
    return mags, 0x80


def _brute_force_codes(y, fmt):
    """Nearest grid magnitude, ties to the even code, sign copied from y."""
    mags, sb = _grid(fmt)
    a = np.abs(y)[:, None]
    dist = np.abs(a - mags[None, :])
    dmin = dist.min(axis=1, keepdims=True)
    cand = dist == dmin
    idx = np.arange(mags.size)[None, :]
    even_pref = np.where(cand & (idx % 2 == 0), idx, 10**6).min(axis=1)
    first = np.where(cand, idx, 10**6).min(axis=1)
    ncand = cand.sum(axis=1)
    code = np.where(ncand > 1, even_pref, first)
    return (code | np.where(np.signbit(y), sb, 0)).astype(np.uint8)


# (amax placed in the group, expected shared exponent X) worked by hand
EXHAUSTIVE_CASES = {
    oracle.E2M1: [(1.0, -2), (6.0, 0), (7.5, 0), (2.0 ** -130, -127), (3.3895313892515355e38, 125), (0.09375, -6)],
    oracle.E4M3: [(1.0, -8), (448.0, 0), (480.0, 0), (2.0 ** -125, -127), (3.3895313892515355e38, 119), (0.09375, -12)],
}


@pytest.mark.parametrize("fmt", [oracle.E2M1, oracle.E4M3])
def test_exhaustive_bf16_encoder(fmt):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bf16_bits_to_f64(allbits)
    finite = np.isfinite(vals)
    for amax, X in EXHAUSTIVE_CASES[fmt]:
        abits = f32_to_bf16_bits(np.float32(amax))
        A = bf16_bits_to_f64(abits)
        sel = finite & (np.abs(vals) <= A)
        xs = allbits[sel]
        rows = np.zeros((xs.size, 32), dtype=np.uint16)
        rows[:, 0] = abits
        rows[:, 7] = xs
        codes, scales = oracle.quantize_rows(rows, fmt)
        assert np.all(scales[:, 0] == X + 127)
        y = vals[sel] * (2.0 ** -X)
        expect = _brute_force_codes(y, fmt)
        got = codes[:, 7]
        bad = np.nonzero(got != expect)[0]
        assert bad.size == 0, (fmt, amax, xs[bad[:5]], got[bad[:5]], expect[bad[:5]])


@pytest.mark.parametrize("fmt", [oracle.E2M1, oracle.E4M3])
def test_quantize_dequantize_idempotent(fmt):
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((4096, 32)) * np.exp2(rng.integers(-20, 20, size=(4096, 1)))).astype(np.float32)
    bits = f32_to_bf16_bits(x)
    c1, s1 = oracle.quantize_rows(bits, fmt)
    deq = oracle.dequantize_rows(c1, s1, fmt)
    bits2 = f32_to_bf16_bits(deq.astype(np.float32))
    assert np.array_equal(bf16_bits_to_f64(bits2), deq)  # the dequantized values are bf16-exact here
    c2, s2 = oracle.quantize_rows(bits2, fmt)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1, c2)


def test_v_tail_group_and_padding():
    """Partial trailing group: amax over valid tokens only; padding codes/scales 0."""
    T = 70
    x = np.zeros((1, T), dtype=np.uint16)
    x[0, :64] = f32_to_bf16_bits(np.full(64, 0.5, np.float32))
    x[0, 64:66] = f32_to_bf16_bits(np.array([3.0, -1.0], np.float32))
    x[0, 66:] = f32_to_bf16_bits(np.full(4, 1000.0, np.float32))  # beyond valid length: ignored
    c, s = oracle.quantize_rows(x, oracle.E4M3, valid=np.array([66], np.int32))
    assert s[0, 2] == 1 - 8 + 127  # amax 3 -> floor(log2 3) = 1
    assert np.all(c[0, 66:] == 0)
    x2 = x.copy()
    c2, s2 = oracle.quantize_rows(x2, oracle.E4M3, valid=np.array([20], np.int32))
    assert s2[0, 1] == 0 and s2[0, 2] == 0 and np.all(c2[0, 20:] == 0)


def test_pack_nibble_order():
    codes = np.array([[1, 2, 3, 4, 15, 0]], dtype=np.uint8)
    assert oracle.pack_e2m1(codes).tolist() == [[0x21, 0x43, 0x0F]]


# ------------------------------------------------------------- attention pins

def deq_e2m1(codes, scales):
    v = E2M1_MAG[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    return v * np.exp2(np.repeat(scales.astype(np.float64) - 127, 32, axis=-1)[..., :codes.shape[-1]])


def deq_e4m3(codes, scales):
    v = E4M3_ALL[codes]
    return v * np.exp2(np.repeat(scales.astype(np.float64) - 127, 32, axis=-1)[..., :codes.shape[-1]])


def naive_attention(q, k, v, seqlens, causal, scale):
    """Softmax attention from the definition. q [B,Sq,Hq,d]; k, v [B,Lk,Hkv,d]."""
    B, Sq, Hq, d = q.shape
    Hkv = k.shape[2]
    out = np.zeros((B, Sq, Hq, d))
    lse = np.full((B, Sq, Hq), -np.inf)
    for b in range(B):
        L = int(seqlens[b])
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            for i in range(Sq):
                n = min(L, i + L - Sq + 1) if causal else L
                if n <= 0:
                    continue
                s = scale * (k[b, :n, hk, :] @ q[b, i, h, :])
                m = s.max()
                p = np.exp(s - m)
                out[b, i, h] = (p @ v[b, :n, hk, :]) / p.sum()
                lse[b, i, h] = m + np.log(p.sum())
    return out, lse


def run_oracle(gen, causal, scale=None):
    qz = oracle.quantize_workload(gen)
    out, lse = oracle.attention(qz["qc"], qz["qs"], qz["kc"], qz["ks"], qz["vc"], qz["vs"],
                                gen["seqlens"], causal=causal, scale=scale)
    return out, lse, qz


def dequantized_inputs(qz):
    qd = np.transpose(deq_e2m1(qz["qc"], qz["qs"]), (0, 2, 1, 3))
    kd = np.transpose(deq_e2m1(qz["kc"], qz["ks"]), (0, 2, 1, 3))
    vd = np.transpose(deq_e4m3(qz["vc"], qz["vs"]), (0, 3, 1, 2))
    return qd, kd, vd


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Lk,causal,lens", [
    (1, 1, 1, 5, 5, True, None),
    (2, 4, 2, 3, 7, True, [7, 4]),
    (2, 6, 2, 8, 8, False, [8, 3]),
    (1, 8, 1, 1, 40, True, [33]),
    (3, 4, 4, 2, 70, True, [70, 1, 35]),
    (1, 2, 1, 6, 6, True, [0]),
])
def test_oracle_matches_naive_on_dequantized(B, Hq, Hkv, Sq, Lk, causal, lens):
    rng = np.random.default_rng(B * 100 + Hq * 10 + Lk)
    gen = dict(q=f32_to_bf16_bits(rng.standard_normal((B, Sq, Hq, 128)).astype(np.float32) * 2),
               k=f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32) * 2),
               v=f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32)),
               seqlens=np.array(lens if lens else [Lk] * B, dtype=np.int32))
    out, lse, qz = run_oracle(gen, causal)
    qd, kd, vd = dequantized_inputs(qz)
    ref, rlse = naive_attention(qd, kd, vd, gen["seqlens"], causal, 1 / math.sqrt(128))
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
    assert np.array_equal(np.isinf(lse), np.isinf(rlse))
    fin = np.isfinite(rlse)
    assert np.allclose(lse[fin], rlse[fin], rtol=0, atol=1e-12)


def _grid_tensor(rng, shape, fmt):
    """Random tensor whose groups of 32 (last axis) are already on the MX grid:
    code * 2^X with one element of magnitude 2^(X + emax) to pin X."""
    if fmt == oracle.E2M1:
        vals = E2M1_MAG
        emax = 2
    else:
        vals = E4M3_ALL[:127]
        emax = 8
    g = rng.choice(vals, size=shape) * rng.choice([-1.0, 1.0], size=shape)
    X = rng.integers(-6, 4, size=shape[:-1] + (shape[-1] // 32,))
    g = g.reshape(shape[:-1] + (shape[-1] // 32, 32))
    g[..., 0] = 2.0 ** emax
    g = g * np.exp2(X)[..., None]
    return g.reshape(shape)


def test_grid_representable_inputs_equal_unquantized_attention():
    rng = np.random.default_rng(5)
    B, Sq, Hq, Hkv, Lk = 2, 5, 4, 2, 64
    q = _grid_tensor(rng, (B, Sq, Hq, 128), oracle.E2M1)
    k = _grid_tensor(rng, (B, Lk, Hkv, 128), oracle.E2M1)
    # V groups run along tokens: build on [B, Hkv, d, Lk] and transpose back.
    v = np.transpose(_grid_tensor(rng, (B, Hkv, 128, Lk), oracle.E4M3), (0, 3, 1, 2))
    for t in (q, k, v):  # every value is exactly a bf16
        assert np.array_equal(bf16_bits_to_f64(f32_to_bf16_bits(t.astype(np.float32))), t)
    gen = dict(q=f32_to_bf16_bits(q.astype(np.float32)), k=f32_to_bf16_bits(k.astype(np.float32)),
               v=f32_to_bf16_bits(v.astype(np.float32)), seqlens=np.array([64, 50], np.int32))
    scale = 1 / 64.0
    out, lse, _ = run_oracle(gen, True, scale)
    ref, rlse = naive_attention(q, k, v, gen["seqlens"], True, scale)
    assert np.allclose(out, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(lse, rlse, rtol=0, atol=1e-12 * np.abs(rlse).max())


def test_closed_forms():
    rng = np.random.default_rng(9)
    B, Sq, Hq, Lk = 1, 4, 2, 4
    v = rng.standard_normal((B, Lk, 1, 128)).astype(np.float32)
    # Q = 0: uniform weights over the allowed (causal) prefix.
    gen = dict(q=np.zeros((B, Sq, Hq, 128), np.uint16),
               k=f32_to_bf16_bits(rng.standard_normal((B, Lk, 1, 128)).astype(np.float32)),
               v=f32_to_bf16_bits(v), seqlens=np.array([Lk], np.int32))
    out, lse, qz = run_oracle(gen, True)
    _, _, vd = dequantized_inputs(qz)
    for i in range(Sq):
        assert np.allclose(out[0, i, 0], vd[0, :i + 1, 0].mean(axis=0), atol=1e-14)
        assert abs(lse[0, i, 0] - math.log(i + 1)) < 1e-14
    # causal row 0 attends only key 0: output is exactly v[0].
    gen["q"] = f32_to_bf16_bits(rng.standard_normal((B, Sq, Hq, 128)).astype(np.float32))
    out, _, qz = run_oracle(gen, True)
    _, _, vd = dequantized_inputs(qz)
    assert np.array_equal(out[0, 0, 1], vd[0, 0, 0])
    # all keys equal: uniform weights whatever Q is.
    kk = np.repeat(rng.standard_normal((1, 1, 1, 128)).astype(np.float32), Lk, axis=1)
    gen["k"] = f32_to_bf16_bits(kk)
    out, _, qz = run_oracle(gen, False)
    _, _, vd = dequantized_inputs(qz)
    assert np.allclose(out[0, 2, 1], vd[0, :, 0].mean(axis=0), atol=1e-14)
    # one key aligned with q far above the rest: output is that key's value row.
    q1 = np.zeros((B, 1, 1, 128), np.float32)
    q1[..., :32] = 4.0
    k1 = np.zeros((B, Lk, 1, 128), np.float32)
    k1[0, 2, 0, :32] = 4.0
    gen2 = dict(q=f32_to_bf16_bits(q1), k=f32_to_bf16_bits(k1), v=f32_to_bf16_bits(v),
                seqlens=np.array([Lk], np.int32))
    out, _, qz = run_oracle(gen2, False)
    _, _, vd = dequantized_inputs(qz)
    assert np.allclose(out[0, 0, 0], vd[0, 2, 0], atol=1e-9)


def test_identity_v_exposes_softmax_weights():
    """V = identity (token j has a one in channel j): output row = softmax weights."""
    rng = np.random.default_rng(3)
    Lk, Sq, Hq = 100, 7, 3
    v = np.zeros((1, Lk, 1, 128), np.float32)
    v[0, np.arange(Lk), 0, np.arange(Lk)] = 1.0
    gen = dict(q=f32_to_bf16_bits(rng.standard_normal((1, Sq, Hq, 128)).astype(np.float32) * 3),
               k=f32_to_bf16_bits(rng.standard_normal((1, Lk, 1, 128)).astype(np.float32)),
               v=f32_to_bf16_bits(v), seqlens=np.array([90], np.int32))
    out, lse, qz = run_oracle(gen, True)
    qd, kd, _ = dequantized_inputs(qz)
    for h in range(Hq):
        for i in range(Sq):
            w = out[0, i, h]
            assert abs(w.sum() - 1.0) < 1e-12
            n = min(90, i + 90 - Sq + 1)
            assert np.all(w[n:] == 0)
            s = (kd[0, :n, 0] @ qd[0, i, h]) / math.sqrt(128)
            p = np.exp(s - s.max())
            assert np.allclose(w[:n], p / p.sum(), atol=1e-15)


def test_sampled_rows_match_full():
    wl = synth.Workload("t", "decode", B=2, Hq=8, Hkv=2, Sq=3, Lk=96, seed=7, k_outliers=2,
                        q_outliers=True, outlier_mult=16.0, len_range=(40, 96))
    gen = wl.generate()
    out, lse, qz = run_oracle(gen, True)
    sel = np.array([[1, 5, 2], [0, 0, 0], [1, 7, 1], [0, 3, 2]], np.int32)
    o2, l2 = oracle.attention(qz["qc"], qz["qs"], qz["kc"], qz["ks"], qz["vc"], qz["vs"], gen["seqlens"],
                              causal=True, sel=sel)
    for r, (b, h, i) in enumerate(sel):
        assert np.array_equal(o2[r], out[b, i, h])
        assert l2[r] == lse[b, i, h]


# ------------------------------------------------- unquantized reference attention

def naive_attention_window(q, k, v, seqlens, causal, scale, window):
    """Softmax attention from the definition with the draft-block window:
    row i of the Sq-row block sees the last `window` keys before the block and
    every key of the block (causal: only keys up to its own position)."""
    B, Sq, Hq, d = q.shape
    Hkv = k.shape[2]
    out = np.zeros((B, Sq, Hq, d))
    lse = np.full((B, Sq, Hq), -np.inf)
    for b in range(B):
        L = int(seqlens[b])
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            for i in range(Sq):
                keys = [j for j in range(L)
                        if (not causal or j <= i + L - Sq) and (window <= 0 or j >= L - Sq - window)]
                if not keys:
                    continue
                s = scale * (k[b, keys, hk, :] @ q[b, i, h, :])
                m = s.max()
                p = np.exp(s - m)
                out[b, i, h] = (p @ v[b, keys, hk, :]) / p.sum()
                lse[b, i, h] = m + np.log(p.sum())
    return out, lse


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Lk,causal,lens,window", [
    (1, 1, 1, 5, 5, True, None, 0),
    (2, 4, 2, 3, 7, True, [7, 4], 0),
    (2, 6, 2, 8, 8, False, [8, 3], 0),
    (3, 4, 4, 2, 70, True, [70, 1, 35], 0),
    (2, 4, 1, 8, 60, False, [60, 20], 16),
    (2, 4, 2, 8, 90, True, [90, 9], 5),
    (1, 2, 1, 1, 40, False, [40], 1),
])
def test_reference_attention_matches_naive(B, Hq, Hkv, Sq, Lk, causal, lens, window):
    rng = np.random.default_rng(B * 1000 + Hq * 10 + Lk + window)
    q = f32_to_bf16_bits(rng.standard_normal((B, Sq, Hq, 128)).astype(np.float32) * 2)
    k = f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32) * 2)
    v = f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32))
    sl = np.array(lens if lens else [Lk] * B, dtype=np.int32)
    out, lse = oracle.attention_ref(q, k, v, sl, causal=causal, window=window)
    ref, rlse = naive_attention_window(bf16_bits_to_f64(q), bf16_bits_to_f64(k), bf16_bits_to_f64(v), sl, causal,
                                       1 / math.sqrt(128), window)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
    assert np.array_equal(np.isinf(lse), np.isinf(rlse))
    fin = np.isfinite(rlse)
    assert np.allclose(lse[fin], rlse[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,window", [(True, 0), (False, 12), (True, 3)])
def test_windowed_oracle_matches_naive_on_dequantized(causal, window):
    rng = np.random.default_rng(77 + window)
    B, Sq, Hq, Hkv, Lk = 2, 8, 4, 2, 100
    gen = dict(q=f32_to_bf16_bits(rng.standard_normal((B, Sq, Hq, 128)).astype(np.float32) * 2),
               k=f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32) * 2),
               v=f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32)),
               seqlens=np.array([100, 37], dtype=np.int32))
    qz = oracle.quantize_workload(gen)
    out, lse = oracle.attention(qz["qc"], qz["qs"], qz["kc"], qz["ks"], qz["vc"], qz["vs"], gen["seqlens"],
                                causal=causal, window=window)
    qd, kd, vd = dequantized_inputs(qz)
    ref, rlse = naive_attention_window(qd, kd, vd, gen["seqlens"], causal, 1 / math.sqrt(128), window)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
    assert np.allclose(lse, rlse, rtol=0, atol=1e-12)


def test_window_closed_forms():
    """A window of W keys before a one-row block sees exactly W + 1 keys; a window
    at least the sequence length changes nothing."""
    rng = np.random.default_rng(4)
    L = 50
    q = np.zeros((1, 1, 1, 128), np.uint16)  # Q = 0: uniform weights over the visible keys
    k = f32_to_bf16_bits(rng.standard_normal((1, L, 1, 128)).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((1, L, 1, 128)).astype(np.float32))
    sl = np.array([L], np.int32)
    vv = bf16_bits_to_f64(v)
    for W in (1, 7, 49):
        out, lse = oracle.attention_ref(q, k, v, sl, causal=True, window=W)
        assert np.allclose(out[0, 0, 0], vv[0, L - 1 - W:, 0].mean(axis=0), atol=1e-14)
        assert abs(lse[0, 0, 0] - math.log(W + 1)) < 1e-13
    o1, l1 = oracle.attention_ref(q, k, v, sl, causal=True, window=L)
    o0, l0 = oracle.attention_ref(q, k, v, sl, causal=True, window=0)
    assert np.array_equal(o1, o0) and np.array_equal(l1, l0)


def test_grid_inputs_quantized_oracle_equals_reference():
    """On MX-grid inputs quantization is the identity, so the quantized oracle and
    the unquantized reference must agree (pins one against the other)."""
    rng = np.random.default_rng(6)
    B, Sq, Hq, Hkv, Lk = 2, 4, 4, 2, 96
    q = _grid_tensor(rng, (B, Sq, Hq, 128), oracle.E2M1)
    k = _grid_tensor(rng, (B, Lk, Hkv, 128), oracle.E2M1)
    v = np.transpose(_grid_tensor(rng, (B, Hkv, 128, Lk), oracle.E4M3), (0, 3, 1, 2))
    gen = dict(q=f32_to_bf16_bits(q.astype(np.float32)), k=f32_to_bf16_bits(k.astype(np.float32)),
               v=f32_to_bf16_bits(v.astype(np.float32)), seqlens=np.array([96, 70], np.int32))
    out, lse, _ = run_oracle(gen, True, 1 / 64.0)
    ref, rlse = oracle.attention_ref(gen["q"], gen["k"], gen["v"], gen["seqlens"], causal=True, scale=1 / 64.0)
    assert np.allclose(out, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(lse, rlse, rtol=0, atol=1e-12 * np.abs(rlse).max())


# ------------------------------------------------------------ Hadamard rotation

def hadamard_matrix(n=128):
    """Sylvester Hadamard matrix from its closed form H[i][j] = (-1)^popcount(i & j)."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    pc = np.vectorize(lambda x: bin(int(x)).count("1"))(i & j)
    return np.where(pc % 2 == 0, 1.0, -1.0)


RSQRT128_F32 = np.float32(2.0 ** -3.5)  # fp32 nearest to 1/sqrt(128)


def test_hadamard_matrix_is_orthogonal():
    H = hadamard_matrix()
    assert np.array_equal(H @ H.T, 128 * np.eye(128))


def test_hadamard_one_hot_rows():
    """x = e_j gives c * (row j of H): every entry +-c with the popcount sign."""
    H = hadamard_matrix()
    for j in (0, 1, 5, 64, 127):
        x = np.zeros((1, 128), np.uint16)
        x[0, j] = f32_to_bf16_bits(np.float32(1.0))
        y = oracle.hadamard_rows(x)[0]
        assert np.array_equal(y, (H[j] * RSQRT128_F32).astype(np.float32)), j


def test_hadamard_integer_inputs_exact():
    """Small integers sum exactly in fp32, so the transform equals the integer
    matrix product, rounded once by the final fp32 multiply."""
    rng = np.random.default_rng(12)
    H = hadamard_matrix()
    xi = rng.integers(-100, 101, size=(64, 128))
    y = oracle.hadamard_rows(f32_to_bf16_bits(xi.astype(np.float32)))
    expect = (xi @ H.T).astype(np.float32) * RSQRT128_F32
    assert np.array_equal(y, expect)


def test_hadamard_random_inputs_within_fp32_bound():
    rng = np.random.default_rng(13)
    H = hadamard_matrix()
    x = rng.standard_normal((256, 128)) * np.exp2(rng.integers(-8, 8, size=(256, 128)))
    bits = f32_to_bf16_bits(x.astype(np.float32))
    xb = bf16_bits_to_f64(bits)
    y = oracle.hadamard_rows(bits).astype(np.float64)
    exact = xb @ H.T / math.sqrt(128)
    # seven butterfly stages and one multiply, each within 2^-24 relative of a partial sum <= sum|x|
    bound = 9 * 2.0 ** -24 * np.abs(xb).sum(axis=1, keepdims=True)
    assert np.all(np.abs(y - exact) <= bound)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(xb, axis=1), rtol=1e-6)


def test_quantize_rows_f32_brute_force():
    """The fp32-input quantizer against the numpy nearest-grid search, on values
    that are not bf16 (rotated rows are general fp32)."""
    rng = np.random.default_rng(14)
    for fmt in (oracle.E2M1, oracle.E4M3):
        x = (rng.standard_normal((2048, 32)) * np.exp2(rng.integers(-30, 30, size=(2048, 1)))).astype(np.float32)
        x[::7, 3] = 0.0
        x[::11] = 0.0
        codes, scales = oracle.quantize_rows_f32(x, fmt)
        emax = 2 if fmt == oracle.E2M1 else 8
        amax = np.abs(x.astype(np.float64)).max(axis=1)
        _, e = np.frexp(amax)
        X = np.where(amax > 0, np.clip(e - 1 - emax, -127, 127), -127)
        assert np.array_equal(scales[:, 0].astype(np.int64), X + 127)
        y = x.astype(np.float64) * np.exp2(-X)[:, None]
        expect = _brute_force_codes(y.ravel(), fmt).reshape(y.shape)
        assert np.array_equal(codes, expect)


def test_quantize_rows_f32_equals_bf16_path_on_bf16_values():
    rng = np.random.default_rng(15)
    bits = f32_to_bf16_bits((rng.standard_normal((512, 128)) * 3).astype(np.float32))
    for fmt in (oracle.E2M1, oracle.E4M3):
        c1, s1 = oracle.quantize_rows(bits, fmt)
        c2, s2 = oracle.quantize_rows_f32(bf16_bits_to_f64(bits).astype(np.float32), fmt)
        assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_rotation_leaves_unquantized_attention_unchanged():
    """(qR).(kR) = q.k: unquantized attention over rotated Q and K equals the
    unrotated one up to the fp32 rounding of the rotation."""
    rng = np.random.default_rng(16)
    B, Sq, Hq, Hkv, Lk = 2, 6, 4, 2, 80
    q = f32_to_bf16_bits(rng.standard_normal((B, Sq, Hq, 128)).astype(np.float32))
    k = f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32))
    sl = np.array([80, 33], np.int32)
    base, blse = oracle.attention_ref(q, k, v, sl, causal=True)
    rot, rlse = oracle.attention_ref(oracle.hadamard_rows(q), oracle.hadamard_rows(k), v, sl, causal=True)
    assert np.abs(rot - base).max() < 1e-5
    assert np.abs(rlse - blse).max() < 1e-5


def test_rotation_spreads_an_outlier_channel():
    """A channel 16x larger than the rest dominates its MX group; after the
    rotation it is spread over every group, so the rotated row's quantization
    error of the non-outlier content is smaller (the article's reason for it)."""
    rng = np.random.default_rng(17)
    x = rng.standard_normal((512, 128)).astype(np.float32)
    x[:, 5] *= 16.0
    bits = f32_to_bf16_bits(x)
    xb = bf16_bits_to_f64(bits)
    c, s = oracle.quantize_rows(bits, oracle.E2M1)
    err_plain = np.abs(oracle.dequantize_rows(c, s, oracle.E2M1) - xb)
    y = oracle.hadamard_rows(bits)
    cr, sr = oracle.quantize_rows_f32(y, oracle.E2M1)
    H = hadamard_matrix()
    back = oracle.dequantize_rows(cr, sr, oracle.E2M1) @ H / math.sqrt(128)  # rotate back
    err_rot = np.abs(back - xb)
    assert err_rot[:, 0:32].mean() < 0.7 * err_plain[:, 0:32].mean()


# ------------------------------------------------------- QK4V4 (V in MXFP4)

@pytest.mark.parametrize("causal,lens", [(True, [70, 33]), (False, [64, 1])])
def test_qk4v4_oracle_matches_naive_on_dequantized(causal, lens):
    """V quantized to E2M1 along tokens (the QK4V4 comparison point): the oracle
    must equal naive attention over the E2M1-dequantized values."""
    rng = np.random.default_rng(40 + len(lens))
    B, Sq, Hq, Hkv, Lk = 2, 3, 4, 2, 70
    gen = dict(q=f32_to_bf16_bits(rng.standard_normal((B, Sq, Hq, 128)).astype(np.float32) * 2),
               k=f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32) * 2),
               v=f32_to_bf16_bits(rng.standard_normal((B, Lk, Hkv, 128)).astype(np.float32)),
               seqlens=np.array(lens, dtype=np.int32))
    qz = oracle.quantize_workload(gen, v_fmt=oracle.E2M1)
    assert qz["vc"].max() <= 15
    out, lse = oracle.attention(qz["qc"], qz["qs"], qz["kc"], qz["ks"], qz["vc"], qz["vs"], gen["seqlens"],
                                causal=causal, v_fmt=oracle.E2M1)
    qd = np.transpose(deq_e2m1(qz["qc"], qz["qs"]), (0, 2, 1, 3))
    kd = np.transpose(deq_e2m1(qz["kc"], qz["ks"]), (0, 2, 1, 3))
    vd = np.transpose(deq_e2m1(qz["vc"], qz["vs"]), (0, 3, 1, 2))
    ref, rlse = naive_attention(qd, kd, vd, gen["seqlens"], causal, 1 / math.sqrt(128))
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
    fin = np.isfinite(rlse)
    assert np.allclose(lse[fin], rlse[fin], rtol=0, atol=1e-12)


def test_qk4v4_grid_inputs_equal_reference():
    rng = np.random.default_rng(41)
    B, Sq, Hq, Hkv, Lk = 1, 4, 2, 1, 64
    q = _grid_tensor(rng, (B, Sq, Hq, 128), oracle.E2M1)
    k = _grid_tensor(rng, (B, Lk, Hkv, 128), oracle.E2M1)
    v = np.transpose(_grid_tensor(rng, (B, Hkv, 128, Lk), oracle.E2M1), (0, 3, 1, 2))
    gen = dict(q=f32_to_bf16_bits(q.astype(np.float32)), k=f32_to_bf16_bits(k.astype(np.float32)),
               v=f32_to_bf16_bits(v.astype(np.float32)), seqlens=np.array([64], np.int32))
    qz = oracle.quantize_workload(gen, v_fmt=oracle.E2M1)
    out, _ = oracle.attention(qz["qc"], qz["qs"], qz["kc"], qz["ks"], qz["vc"], qz["vs"], gen["seqlens"],
                              causal=True, scale=1 / 64.0, v_fmt=oracle.E2M1)
    ref, _ = oracle.attention_ref(gen["q"], gen["k"], gen["v"], gen["seqlens"], causal=True, scale=1 / 64.0)
    assert np.allclose(out, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_qk4v4_error_exceeds_qk4v8_error():
    """V at 4 bits loses more than V at 8 bits (the article's section 2.2): with
    Q and K quantized the same way, the error that V's quantization adds to the
    output (against the same attention over unquantized V) is several times
    larger for E2M1 than for E4M3."""
    wl = synth.Workload("t", "decode", B=2, Hq=8, Hkv=2, Sq=4, Lk=300, seed=5)
    gen = wl.generate()
    errs = {}
    for fmt in (oracle.E4M3, oracle.E2M1):
        qz = oracle.quantize_workload(gen, v_fmt=fmt)
        o, _ = oracle.attention(qz["qc"], qz["qs"], qz["kc"], qz["ks"], qz["vc"], qz["vs"], gen["seqlens"],
                                causal=True, v_fmt=fmt)
        qd = np.transpose(deq_e2m1(qz["qc"], qz["qs"]), (0, 2, 1, 3))
        kd = np.transpose(deq_e2m1(qz["kc"], qz["ks"]), (0, 2, 1, 3))
        ref, _ = naive_attention(qd, kd, bf16_bits_to_f64(gen["v"]), gen["seqlens"], True, 1 / math.sqrt(128))
        errs[fmt] = np.abs(o - ref).mean()
    assert errs[oracle.E2M1] > 3 * errs[oracle.E4M3]
