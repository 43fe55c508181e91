"""Bit-exact MX quantization on the GPU against the CPU oracle.

Packed codes and E8M0 scales have exactly one correct value. Every case
compares them byte for byte after rearranging the library's layout into the
oracle's logical order.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import oracle
import synth
from gpu_util import to_dev
from layouts import qk_scales_logical, unpack_e2m1, v_codes_logical, v_scales_logical

pytestmark = pytest.mark.gpu


def f32_to_bf16_bits(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def check_qk(bits, cap=None, seqlens=None):
    B, T, H, _ = bits.shape
    sl = None if seqlens is None else torch.tensor(list(seqlens), dtype=torch.int32)
    xp = qk.quantize_qk(to_dev(bits), cap=cap, seqlens=sl)
    torch.cuda.synchronize()
    codes = xp.codes.cpu().numpy()
    scales = xp.scales.cpu().numpy()
    oc, os_ = oracle.quantize_qk(bits)
    if seqlens is not None:
        for b in range(B):
            oc[b, :, seqlens[b]:] = 0
            os_[b, :, seqlens[b]:] = 0
    assert np.array_equal(unpack_e2m1(codes[:, :, :T]), oc)
    assert np.array_equal(qk_scales_logical(scales, T), os_)
    assert not codes[:, :, T:].any()
    assert not qk_scales_logical(scales, xp.cap)[:, :, T:].any()


def check_v(bits, cap=None, seqlens=None):
    B, T, H, _ = bits.shape
    sl = None if seqlens is None else torch.tensor(seqlens, dtype=torch.int32)
    vp = qk.quantize_v(to_dev(bits), cap=cap, seqlens=sl)
    torch.cuda.synchronize()
    codes = v_codes_logical(vp.codes.cpu().numpy())
    scales = vp.scales.cpu().numpy()
    oc, os_ = oracle.quantize_v(bits, seqlens)
    assert np.array_equal(codes[..., :T], oc)
    assert np.array_equal(v_scales_logical(scales, T), os_)
    assert not codes[..., T:].any()
    nG = (T + 31) // 32
    assert not v_scales_logical(scales, vp.cap)[..., nG:].any()


# Group maxima chosen to pin the shared exponent, including both clamps and
# the saturating ranges (worked by hand: X = floor(log2 amax) - emax).
AMAXES = [1.0, 6.0, 7.5, 448.0, 480.0, 2.0 ** -130, 3.3895313892515355e38, 0.09375]


@pytest.mark.parametrize("amax", AMAXES)
def test_qk_exhaustive_bf16(amax):
    """Every finite bf16 x with |x| <= amax, quantized inside a group whose max is amax."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (allbits.astype(np.uint32) << 16).view(np.float32)
    abits = f32_to_bf16_bits(np.float32(amax))
    A = (np.uint32(abits) << 16).view(np.float32)
    xs = allbits[np.isfinite(vals) & (np.abs(vals) <= A)]
    n = xs.size
    rows = np.zeros((1, n, 1, 128), dtype=np.uint16)
    rows[0, :, 0, 0] = abits          # group 0 holds [A, ..., x, ...]
    rows[0, :, 0, 7] = xs
    rows[0, :, 0, 40] = xs            # group 1: x is its own max
    rows[0, :, 0, 64 + 3] = abits     # group 2: A alone
    check_qk(rows)


@pytest.mark.parametrize("amax", AMAXES)
def test_v_exhaustive_bf16(amax):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (allbits.astype(np.uint32) << 16).view(np.float32)
    abits = f32_to_bf16_bits(np.float32(amax))
    A = (np.uint32(abits) << 16).view(np.float32)
    xs = allbits[np.isfinite(vals) & (np.abs(vals) <= A)]
    n_groups = (xs.size + 127) // 128
    xs = np.concatenate([xs, np.zeros(n_groups * 128 - xs.size, np.uint16)])
    T = 32 * n_groups
    v = np.zeros((1, T, 1, 128), dtype=np.uint16)
    grid = xs.reshape(n_groups, 128)
    v[0, 32 * np.arange(n_groups), 0, :] = abits
    v[0, 32 * np.arange(n_groups) + 7, 0, :] = grid
    check_v(v)


@pytest.mark.parametrize("B,T,H,cap", [(1, 1, 1, 128), (2, 37, 3, 128), (1, 129, 2, 384), (3, 300, 2, 384)])
def test_qk_random_shapes(B, T, H, cap):
    rng = np.random.default_rng(T)
    x = rng.standard_normal((B, T, H, 128)).astype(np.float32) * np.exp2(rng.integers(-8, 8, (B, T, H, 1)))
    check_qk(f32_to_bf16_bits(x), cap=cap)


def test_qk_strided_input_and_seqlens():
    rng = np.random.default_rng(1)
    full = f32_to_bf16_bits(rng.standard_normal((2, 50, 6, 128)).astype(np.float32))
    dev = to_dev(full)[:, :, 1:4, :]       # non-contiguous head slice
    xp = qk.quantize_qk(dev, cap=128, seqlens=torch.tensor([50, 20], dtype=torch.int32))
    oc, os_ = oracle.quantize_qk(np.ascontiguousarray(full[:, :, 1:4, :]))
    oc[1, :, 20:] = 0
    os_[1, :, 20:] = 0
    assert np.array_equal(unpack_e2m1(xp.codes.cpu().numpy()[:, :, :50]), oc)
    assert np.array_equal(qk_scales_logical(xp.scales.cpu().numpy(), 50), os_)


@pytest.mark.parametrize("T,lens", [(1, None), (31, None), (33, None), (127, None), (129, None), (200, [200, 70]),
                                    (256, [1, 255])])
def test_v_random_shapes_and_tails(T, lens):
    B = 1 if lens is None else len(lens)
    rng = np.random.default_rng(T)
    x = rng.standard_normal((B, T, 2, 128)).astype(np.float32) * np.exp2(rng.integers(-8, 8, (B, T, 1, 128)))
    check_v(f32_to_bf16_bits(x), seqlens=lens)


def test_v_padding_poison_ignored():
    """Tokens past seqlens hold NaN bf16; they must not reach any code or scale."""
    wl = synth.Workload("t", "decode", B=2, Hq=2, Hkv=2, Sq=1, Lk=256, seed=3, len_range=(100, 200))
    gen = wl.generate(pad_bits=0x7FC0)
    check_v(gen["v"], seqlens=list(gen["seqlens"]))
    check_qk(gen["k"], seqlens=list(gen["seqlens"]))


@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER)
def test_workload_quantize_bit_exact(name):
    """Full-size workloads: Q, K, V packed bytes bit-exact (large ones on 2 batches)."""
    wl = synth.WORKLOADS[name]
    gen = wl.generate()
    lens = gen["seqlens"]
    sl = torch.from_numpy(lens).cuda()
    qp = qk.quantize_qk(to_dev(gen["q"]))
    kp = qk.quantize_qk(to_dev(gen["k"]), seqlens=sl)
    vp = qk.quantize_v(to_dev(gen["v"]), seqlens=sl)
    torch.cuda.synchronize()
    bsel = list(range(wl.B)) if wl.B * wl.Lk * wl.Hkv <= 32 * 8192 * 8 else [0, wl.B - 1]
    for b in bsel:
        oc, os_ = oracle.quantize_qk(gen["q"][b:b + 1])
        assert np.array_equal(unpack_e2m1(qp.codes[b:b + 1].cpu().numpy()[:, :, :wl.Sq]), oc)
        assert np.array_equal(qk_scales_logical(qp.scales[b:b + 1].cpu().numpy(), wl.Sq), os_)
        kc, ks = oracle.quantize_qk(gen["k"][b:b + 1])
        assert np.array_equal(unpack_e2m1(kp.codes[b:b + 1].cpu().numpy()[:, :, :wl.Lk]), kc)
        assert np.array_equal(qk_scales_logical(kp.scales[b:b + 1].cpu().numpy(), wl.Lk), ks)
        vc, vs = oracle.quantize_v(gen["v"][b:b + 1], lens[b:b + 1])
        assert np.array_equal(v_codes_logical(vp.codes[b:b + 1].cpu().numpy())[..., :wl.Lk], vc)
        assert np.array_equal(v_scales_logical(vp.scales[b:b + 1].cpu().numpy(), wl.Lk), vs)


@pytest.mark.timeout(300)
def test_qk_batch_beyond_grid_y_limit():
    """B = 65537 sequences: the launcher runs the batch in chunks of 65535 grid
    rows, offsetting inputs, lengths, codes and scales per chunk. Entries on both
    sides of the chunk boundary and the last one must match the oracle."""
    B = 65537
    rng = np.random.default_rng(21)
    bits = f32_to_bf16_bits(rng.standard_normal((B, 1, 1, 128)).astype(np.float32) * 4)
    lens = np.ones((B,), np.int32)
    lens[65535] = 0   # first entry of the second chunk is empty
    xp = qk.quantize_qk(to_dev(bits), cap=128, seqlens=torch.from_numpy(lens).cuda())
    torch.cuda.synchronize()
    oc, os_ = oracle.quantize_qk(bits)
    oc[lens == 0] = 0
    os_[lens == 0] = 0
    for b in (0, 1, 65534, 65535, 65536):
        codes = xp.codes[b].cpu().numpy()
        scales = xp.scales[b].cpu().numpy()
        assert np.array_equal(unpack_e2m1(codes[None, :, :1])[0], oc[b]), b
        assert np.array_equal(qk_scales_logical(scales[None], 1)[0], os_[b]), b
        assert not codes[:, 1:].any()
