"""Draft-block attention (sliding window) on the GPU against the fp64 oracle.

With a window W, every query row of the nq-token block at the end of a
sequence of L keys sees only keys j >= L - nq - W (the last W keys before the
block, and the block), non-causal in the block as in the DFlash draft model, or
causal. The cases cover both split kernels that take a window (up to 32 query
rows per KV head, and 33..64), windows whose first key falls in either half of
its 128-key tile (the GQA kernel takes its reference maximum from the first
half holding a visible key), one and several splits, ragged lengths, windows
wider than the sequence, and the bf16-query entry point.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import oracle
import synth
from gpu_util import assert_close, quantize_on_gpu, to_dev
from layouts import fill_v_bytes

pytestmark = pytest.mark.gpu


def _gen(B, Hq, Hkv, nq, lens, seed, k_out=4):
    Lk = max(lens)
    wl = synth.Workload("w", "decode", B=B, Hq=Hq, Hkv=Hkv, Sq=nq, Lk=Lk, seed=seed, k_outliers=k_out,
                        q_outliers=k_out > 0, outlier_mult=16.0)
    gen = wl.generate()
    gen["seqlens"] = np.array(lens, dtype=np.int32)
    for b, L in enumerate(lens):
        gen["k"][b, L:] = 0
        gen["v"][b, L:] = 0
    return gen


def _oracle(gen, causal, window):
    oz = oracle.quantize_workload(gen)
    return oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], gen["seqlens"],
                            causal=causal, window=window)


@pytest.mark.parametrize("Hq,Hkv,nq,causal,window,splits,lens", [
    (32, 8, 1, True, 1024, 0, [2000, 1200, 700, 5000]),      # 4 rows: swap-AB kernel
    (16, 4, 8, False, 1024, 0, [2008, 1508, 1208]),          # 32 rows, non-causal draft block
    (16, 4, 8, False, 300, 3, [2000, 999, 4000]),            # several splits inside the window
    (64, 8, 8, False, 1024, 0, [2000, 1500, 1200, 5008]),     # 64 rows: GQA kernel; lo % 128 = 72, 84, 40, ...
    (64, 8, 8, True, 1024, 2, [2000, 1500, 3000]),            # GQA kernel, causal block, two splits
    (48, 8, 8, False, 100, 4, [1000, 777, 129, 64]),          # window narrower than a tile; L < nq + window
    (64, 8, 8, False, 5000, 0, [1000, 300]),                  # window wider than the sequence
])
def test_window_decode_matches_oracle(Hq, Hkv, nq, causal, window, splits, lens):
    gen = _gen(len(lens), Hq, Hkv, nq, lens, seed=sum(lens) % 1000 + Hq)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    out, lse = qk.attention_decode(qp, kp, vp, sl, max_seqlen=max(lens), causal_in_block=causal, num_splits=splits,
                                   window=window, return_lse=True)
    torch.cuda.synchronize()
    ref, rlse = _oracle(gen, causal, window)
    assert_close(out, ref, f"window {window} Hq={Hq} nq={nq} causal={causal}")
    got = np.transpose(lse.cpu().numpy(), (0, 2, 1))
    assert np.abs(got - rlse).max() < 1e-2


@pytest.mark.parametrize("Hq,Hkv,nq,window", [(32, 8, 1, 1024), (16, 2, 8, 1024), (64, 8, 8, 1024)])
def test_window_decode_bf16_queries(Hq, Hkv, nq, window):
    lens = [3000, 2100, 1100]
    gen = _gen(len(lens), Hq, Hkv, nq, lens, seed=Hq + nq)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    out = qk.attention_decode_bf16(to_dev(gen["q"]), kp, vp, sl, max_seqlen=max(lens), causal_in_block=False,
                                   window=window)
    packed = qk.attention_decode(qp, kp, vp, sl, max_seqlen=max(lens), causal_in_block=False, window=window)
    torch.cuda.synchronize()
    ref, _ = _oracle(gen, False, window)
    assert_close(out, ref, f"bf16 window Hq={Hq} nq={nq}")
    assert_close(packed, ref, f"packed window Hq={Hq} nq={nq}")


def test_window_streams_only_the_window():
    """Keys before the window's first tile are never read: poisoning them with
    NaN patterns leaves the output unchanged, bit for bit."""
    lens = [4000, 3000]
    W, nq = 1024, 8
    gen = _gen(2, 64, 8, nq, lens, seed=5)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    clean = qk.attention_decode(qp, kp, vp, sl, max_seqlen=4000, causal_in_block=False, window=W)
    torch.cuda.synchronize()
    clean = clean.clone()
    for b, L in enumerate(lens):
        t0 = (L - nq - W) // 128          # first tile of the window
        kp.codes[b, :, :t0 * 128] = 0xFF
        fill_v_bytes(vp.codes, b, 0, 0xFF, stop=t0 * 128)
        kp.scales[b, :, :t0] = 0xFF
        vp.scales[b, :, :t0] = 0xFF
    dirty = qk.attention_decode(qp, kp, vp, sl, max_seqlen=4000, causal_in_block=False, window=W)
    torch.cuda.synchronize()
    assert torch.equal(clean, dirty)


def test_window_rejected_for_large_groups():
    lens = [500]
    gen = _gen(1, 16, 1, 8, lens, seed=1, k_out=0)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    with pytest.raises(qk.QK4V8Error, match="window"):
        qk.attention_decode(qp, kp, vp, sl, max_seqlen=500, window=64)
