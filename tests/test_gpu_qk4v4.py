"""QK4V4, the MpFA article's comparison point (section 2.2), on the GPU.

qk4v8_quantize_v4 packs V to MXFP4 along tokens; its bytes must equal the
oracle's E2M1 quantization of V exactly. qk4v8_attention_decode_v4 (and the
bf16-query form) run the swap-AB decode kernel with V as the E2M1 operand of the
block-scaled MMA; the output must match the oracle's attention over E2M1 V
within the usual tolerance.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import oracle
import synth
from gpu_util import assert_close, to_dev
from layouts import fill_v_bytes, v_codes_logical, v_scales_logical

pytestmark = pytest.mark.gpu


def f32_to_bf16_bits(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def unpack_tokens(codes):
    """[..., cap/2] bytes -> [..., cap] E2M1 codes, even token in the low nibble."""
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = codes & 0xF
    out[..., 1::2] = codes >> 4
    return out


def check_v4(bits, cap=None, seqlens=None):
    B, T, H, _ = bits.shape
    sl = None if seqlens is None else torch.tensor(list(seqlens), dtype=torch.int32)
    vp = qk.quantize_v4(to_dev(bits), cap=cap, seqlens=sl)
    torch.cuda.synchronize()
    codes = unpack_tokens(v_codes_logical(vp.codes.cpu().numpy()))
    scales = vp.scales.cpu().numpy()
    oc, os_ = oracle.quantize_v(bits, seqlens, fmt=oracle.E2M1)
    assert np.array_equal(codes[..., :T], oc)
    assert np.array_equal(v_scales_logical(scales, T), os_)
    assert not codes[..., T:].any()


@pytest.mark.parametrize("B,T,H,seed", [(1, 1, 1, 0), (2, 300, 3, 1), (3, 129, 8, 2), (1, 1000, 2, 3)])
def test_v4_quantize_matches_oracle(B, T, H, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, T, H, 128)) * np.exp2(rng.integers(-6, 6, size=(B, T, H, 1)))
    check_v4(f32_to_bf16_bits(x.astype(np.float32)))


def test_v4_quantize_lengths_and_amax_edges():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 200, 2, 128)).astype(np.float32)
    x[0, 40, 0, :] = 6.0           # group max exactly at the E2M1 maximum
    x[0, 41, 0, :] = 7.5           # saturates
    x[1, :, 1, :] = 0.0            # all-zero groups
    x[2, 100, 0, 5] = -0.0
    check_v4(f32_to_bf16_bits(x), cap=256, seqlens=[200, 31, 129])


def _gen(B, Hq, Hkv, nq, lens, seed):
    wl = synth.Workload("v4", "decode", B=B, Hq=Hq, Hkv=Hkv, Sq=nq, Lk=max(lens), seed=seed, k_outliers=4,
                        q_outliers=True, outlier_mult=16.0)
    gen = wl.generate()
    gen["seqlens"] = np.array(lens, np.int32)
    for b, L in enumerate(lens):
        gen["k"][b, L:] = 0
        gen["v"][b, L:] = 0
    return gen


@pytest.mark.parametrize("Hq,Hkv,nq,causal,window,splits", [
    (32, 8, 1, True, 0, 1),       # 4 rows, one launch
    (64, 8, 1, True, 0, 0),       # 8 rows (the long-context decode shape)
    (16, 4, 8, True, 0, 3),       # 32 rows, splits + merge
    (64, 8, 8, True, 0, 2),       # 64 rows on the swap-AB kernel
    (16, 2, 8, False, 700, 0),    # draft-block window
])
def test_v4_decode_matches_oracle(Hq, Hkv, nq, causal, window, splits):
    lens = [1500, 700, 1281, 64]
    gen = _gen(len(lens), Hq, Hkv, nq, lens, seed=Hq + nq + splits)
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    qp = qk.quantize_qk(to_dev(gen["q"]))
    kp = qk.quantize_qk(to_dev(gen["k"]), seqlens=sl)
    vp = qk.quantize_v4(to_dev(gen["v"]), seqlens=sl)
    out, lse = qk.attention_decode(qp, kp, vp, sl, max_seqlen=max(lens), causal_in_block=causal, num_splits=splits,
                                   window=window, return_lse=True)
    out16 = qk.attention_decode_bf16(to_dev(gen["q"]), kp, vp, sl, max_seqlen=max(lens), causal_in_block=causal,
                                     num_splits=splits, window=window)
    torch.cuda.synchronize()
    oz = oracle.quantize_workload(gen, v_fmt=oracle.E2M1)
    ref, rlse = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], gen["seqlens"],
                                 causal=causal, window=window, v_fmt=oracle.E2M1)
    assert_close(out, ref, f"QK4V4 decode Hq={Hq} nq={nq}")
    assert_close(out16, ref, f"QK4V4 bf16 decode Hq={Hq} nq={nq}")
    got = np.transpose(lse.cpu().numpy(), (0, 2, 1))
    assert np.abs(got - rlse).max() < 1e-2


def test_v4_decode_poisoned_scales_past_length():
    """V scale bytes of groups past each length set to the E8M0 NaN pattern: the
    kernel zeroes them in shared memory, so the output is unchanged."""
    lens = [300, 45]
    gen = _gen(2, 32, 8, 1, lens, seed=3)
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    qp = qk.quantize_qk(to_dev(gen["q"]))
    kp = qk.quantize_qk(to_dev(gen["k"]), seqlens=sl, cap=512)
    vp = qk.quantize_v4(to_dev(gen["v"]), seqlens=sl, cap=512)
    clean = qk.attention_decode(qp, kp, vp, sl, max_seqlen=300, num_splits=2)
    torch.cuda.synchronize()
    clean = clean.clone()
    for b, L in enumerate(lens):
        blk0 = L // 128
        vp.scales[b, :, blk0 + 1:] = 0xFF
        fill_v_bytes(vp.codes, b, (L + 1) // 2, 0xFF)   # E2M1 -6: finite, and P is zero there
        jv = L - blk0 * 128
        idx = torch.tensor([(c % 32) * 16 + (c // 32) * 4 + g for c in range(128) for g in range((jv + 31) // 32, 4)],
                           dtype=torch.long, device="cuda")
        if idx.numel():
            vp.scales[b, :, blk0, idx] = 0xFF
    dirty = qk.attention_decode(qp, kp, vp, sl, max_seqlen=300, num_splits=2)
    torch.cuda.synchronize()
    assert torch.equal(clean, dirty)
