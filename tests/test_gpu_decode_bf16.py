"""qk4v8_attention_decode_bf16: the decode step from bf16 queries.

The call quantizes the queries itself: inside the split kernel for up to 64
query rows per KV head, or into its workspace for larger groups. It must give
the same bytes as qk4v8_quantize_qk followed by qk4v8_attention_decode, so
the comparison is exact (torch.equal). Parity with the fp64 oracle then
follows from the packed path's parity tests, and is also checked here
directly on two shapes.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import synth
from gpu_util import assert_close, oracle_attention_from, to_dev

pytestmark = pytest.mark.gpu


def make(B, nq, L, Hq, Hkv, seed, lens=None):
    wl = synth.Workload("t", "decode", B=B, Hq=Hq, Hkv=Hkv, Sq=nq, Lk=L, seed=seed, k_outliers=4,
                        q_outliers=True, outlier_mult=16.0)
    gen = wl.generate()
    if lens is not None:
        gen["seqlens"] = np.array(lens, dtype=np.int32)
    q = to_dev(gen["q"])
    sl = torch.from_numpy(gen["seqlens"].astype(np.int32)).cuda()
    kp = qk.quantize_qk(to_dev(gen["k"]), seqlens=sl)
    vp = qk.quantize_v(to_dev(gen["v"]), seqlens=sl)
    return gen, q, kp, vp, sl


def packed_reference(q, kp, vp, sl, L, splits):
    qp = qk.quantize_qk(q)
    return qk.attention_decode(qp, kp, vp, sl, max_seqlen=L, num_splits=splits, return_lse=True)


@pytest.mark.parametrize("B,nq,L,Hq,Hkv,splits,lens", [
    (4, 1, 3000, 32, 8, 1, None),             # 4 rows, one split: the kernel writes out directly
    (4, 1, 3000, 32, 8, 3, None),             # 4 rows, partials and merge
    (2, 8, 2000, 64, 8, 1, [2000, 777]),      # 64 rows (verify block), direct
    (2, 8, 2000, 64, 8, 2, [2000, 777]),      # 64 rows, merge
    (3, 3, 900, 12, 4, 1, [900, 1, 129]),     # odd row count, short sequences
    (2, 8, 700, 128, 8, 2, [700, 300]),       # 128 rows: queries quantized into the workspace
    (2, 8, 700, 128, 8, 1, [700, 300]),
])
def test_bf16_queries_match_packed_path_exactly(B, nq, L, Hq, Hkv, splits, lens):
    gen, q, kp, vp, sl = make(B, nq, L, Hq, Hkv, seed=L + Hq + splits, lens=lens)
    ref, ref_lse = packed_reference(q, kp, vp, sl, L, splits)
    out, lse = qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=L, num_splits=splits, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.equal(lse, ref_lse)


def test_bf16_strided_queries():
    """Queries read through strides: a [B, nq, Hq, 128] view into a wider buffer."""
    gen, q, kp, vp, sl = make(2, 4, 1500, 16, 2, seed=31)
    wide = torch.zeros((2, 4, 24, 256), dtype=torch.bfloat16, device="cuda")
    wide[:, :, 4:20, 64:192] = q
    qv = wide[:, :, 4:20, 64:192]
    assert not qv.is_contiguous()
    for splits in (1, 2):
        ref, _ = packed_reference(q, kp, vp, sl, 1500, splits)
        out = qk.attention_decode_bf16(qv, kp, vp, sl, max_seqlen=1500, num_splits=splits)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


def test_bf16_zero_length_sequence_direct():
    gen, q, kp, vp, sl = make(2, 2, 256, 4, 2, seed=3, lens=[256, 0])
    out, lse = qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=256, num_splits=1, return_lse=True)
    torch.cuda.synchronize()
    assert out[1].float().abs().max().item() == 0
    assert torch.isinf(lse[1]).all() and (lse[1] < 0).all()
    (ref, _), _ = oracle_attention_from(gen, True)
    assert_close(out, ref, "bf16 decode, zero-length sequence")


@pytest.mark.parametrize("B,nq,L,Hq,Hkv,splits", [
    (3, 1, 2500, 32, 8, 1),
    (2, 8, 1200, 64, 8, 0),
])
def test_bf16_decode_oracle_parity(B, nq, L, Hq, Hkv, splits):
    gen, q, kp, vp, sl = make(B, nq, L, Hq, Hkv, seed=7 * L + nq)
    out, lse = qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=L, num_splits=splits, return_lse=True)
    torch.cuda.synchronize()
    (ref, rlse), _ = oracle_attention_from(gen, True)
    assert_close(out, ref, f"bf16 decode B{B} nq{nq} Hq{Hq}")
    l = lse.cpu().numpy().transpose(0, 2, 1)
    assert np.abs(l - rlse).max() < 1e-2


def test_bf16_decode_graph_capture():
    """The call enqueues on the current stream only, so it can be captured in a CUDA graph."""
    gen, q, kp, vp, sl = make(2, 1, 1024, 32, 8, seed=12)
    out = torch.empty((2, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
    qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=1024, num_splits=1, out=out)   # first call outside
    torch.cuda.synchronize()
    ref = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        qk.attention_decode_bf16(q, kp, vp, sl, max_seqlen=1024, num_splits=1, out=out)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
