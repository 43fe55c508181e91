"""Hadamard-rotated Q/K quantization on the GPU against the CPU oracle.

qk4v8_quantize_qk_hadamard rotates each (token, head) row by H/sqrt(128) and
quantizes the rotated values to MXFP4 (MpFA article, sections 2.1 and 3.1). The
rotated values decide the codes, so both sides compute the rotation in fp32
with the same butterfly order, and the packed bytes must match exactly. The
attention over rotated Q and K must then match the oracle's attention over the
oracle's own rotated codes within the usual tolerance.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import oracle
import synth
from gpu_util import assert_close, to_dev
from layouts import qk_scales_logical, unpack_e2m1

pytestmark = pytest.mark.gpu


def f32_to_bf16_bits(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def check_rot(bits, cap=None, seqlens=None, x_dev=None):
    B, T, H, _ = bits.shape
    sl = None if seqlens is None else torch.tensor(list(seqlens), dtype=torch.int32)
    xp = qk.quantize_qk(to_dev(bits) if x_dev is None else x_dev, cap=cap, seqlens=sl, hadamard=True)
    torch.cuda.synchronize()
    codes = xp.codes.cpu().numpy()
    scales = xp.scales.cpu().numpy()
    oc, os_ = oracle.quantize_qk_hadamard(bits, seqlens)
    got_c = unpack_e2m1(codes[:, :, :T])
    got_s = qk_scales_logical(scales, T)
    bad = np.argwhere(got_c != oc)
    assert bad.size == 0, f"{bad.shape[0]} code mismatches, first at {bad[:3].tolist()}"
    assert np.array_equal(got_s, os_)
    assert not codes[:, :, T:].any()
    assert not qk_scales_logical(scales, xp.cap)[:, :, T:].any()
    return xp


@pytest.mark.parametrize("B,T,H,seed", [(1, 1, 1, 0), (2, 300, 3, 1), (3, 129, 8, 2), (1, 1000, 2, 3)])
def test_rotated_quantize_normal(B, T, H, seed):
    rng = np.random.default_rng(seed)
    check_rot(f32_to_bf16_bits(rng.standard_normal((B, T, H, 128)).astype(np.float32)))


def test_rotated_quantize_wide_exponent_range():
    """Inputs spread over 40 binades: the fp32 transform rounds, so this pins the
    butterfly order and the final multiply, not only the grid."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 257, 4, 128)) * np.exp2(rng.integers(-20, 20, size=(2, 257, 4, 128)))
    check_rot(f32_to_bf16_bits(x.astype(np.float32)))


def test_rotated_quantize_outliers_seqlens_and_strides():
    wl = synth.Workload("t", "decode", B=3, Hq=8, Hkv=4, Sq=1, Lk=500, seed=9, k_outliers=4, outlier_mult=20.0,
                        k_dist=synth.DIST_STUDENT_T3)
    gen = wl.generate()
    check_rot(gen["k"], cap=640, seqlens=[500, 3, 257])
    # A strided view: K taken out of a fused [B, T, H, 2, 128] buffer.
    big = np.zeros((3, 500, 4, 2, 128), np.uint16)
    big[:, :, :, 1, :] = gen["k"]
    dev = to_dev(big)[:, :, :, 1, :]
    check_rot(gen["k"], x_dev=dev)


def test_rotated_quantize_zero_and_one_hot_rows():
    bits = np.zeros((1, 130, 2, 128), np.uint16)
    bits[0, 1, 0, 0] = f32_to_bf16_bits(np.float32(1.0))
    bits[0, 2, 1, 127] = f32_to_bf16_bits(np.float32(-3.0))
    bits[0, 3, 0, :] = 0x8000   # -0.0 everywhere
    check_rot(bits)


@pytest.mark.timeout(300)
def test_rotated_quantize_prefill_workload_k():
    """K of the B=4, Hkv=8, S=8192 prefill workload (2 outlier channels x20 per head), whole tensor."""
    gen = synth.WORKLOADS["prefill_gqa_b4_hq32_hkv8_s8192"].generate()
    check_rot(gen["k"])


def _rotated_oracle(gen, causal):
    qc, qs = oracle.quantize_qk_hadamard(gen["q"])
    kc, ks = oracle.quantize_qk_hadamard(gen["k"], gen["seqlens"])
    vc, vs = oracle.quantize_v(gen["v"], gen["seqlens"])
    return oracle.attention(qc, qs, kc, ks, vc, vs, gen["seqlens"], causal=causal)


def test_rotated_prefill_attention_parity():
    wl = synth.Workload("t", "prefill", B=2, Hq=8, Hkv=2, Sq=300, Lk=300, seed=11, k_outliers=2,
                        q_outliers=False, outlier_mult=20.0)
    gen = wl.generate()
    gen["seqlens"] = np.array([300, 170], np.int32)
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    qp, kp, vp = qk.quantize(to_dev(gen["q"]), to_dev(gen["k"]), to_dev(gen["v"]), seqlens_k=sl, hadamard=True)
    out, lse = qk.attention_prefill(qp, kp, vp, seqlens_k=sl, causal=True, return_lse=True)
    torch.cuda.synchronize()
    ref, rlse = _rotated_oracle(gen, causal=True)
    assert_close(out, ref, "rotated prefill")
    fin = np.isfinite(rlse)
    got = np.transpose(lse.cpu().numpy(), (0, 2, 1))
    assert np.abs(got[fin] - rlse[fin]).max() < 1e-2


@pytest.mark.parametrize("Hq,Hkv,nq,splits", [(32, 8, 1, 0), (64, 8, 8, 3), (16, 4, 8, 2)])
def test_rotated_decode_attention_parity(Hq, Hkv, nq, splits):
    wl = synth.Workload("t", "decode", B=3, Hq=Hq, Hkv=Hkv, Sq=nq, Lk=1500, seed=12, k_outliers=4,
                        q_outliers=True, outlier_mult=16.0, len_range=(600, 1500))
    gen = wl.generate()
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    qp = qk.quantize_qk(to_dev(gen["q"]), hadamard=True)
    kp = qk.quantize_qk(to_dev(gen["k"]), seqlens=sl, hadamard=True)
    vp = qk.quantize_v(to_dev(gen["v"]), seqlens=sl)
    out = qk.attention_decode(qp, kp, vp, sl, max_seqlen=int(gen["seqlens"].max()), num_splits=splits)
    torch.cuda.synchronize()
    ref, _ = _rotated_oracle(gen, causal=True)
    assert_close(out, ref, f"rotated decode Hq={Hq} nq={nq}")
