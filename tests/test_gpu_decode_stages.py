"""The two exported decode stages, qk4v8_attention_decode_splitkv and
qk4v8_decode_merge, called one after the other through the C ABI.

The split-KV launch writes each split's normalised partial O and log2-sum-exp
to the caller's workspace; the merge combines them. Their result must match the
fp64 oracle within the attention tolerance, and equal qk4v8_attention_decode
(which runs the same two kernels) bit for bit when that call also merges. All
three split kernels are covered: up to 32 query rows per KV head (swap-AB),
33..64 (GQA decode kernel, fixed-split partials) and 65..128 (128-row kernel).
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import synth
from bit_quantized_attention_qk4v8_b200 import _lib
from gpu_util import assert_close, oracle_attention_from, quantize_on_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hq,Hkv,nq,L,splits,causal", [
    (3, 16, 4, 2, 1500, 3, True),     # 8 rows: swap-AB kernel
    (2, 32, 8, 1, 700, 2, True),      # 4 rows
    (2, 64, 8, 8, 1200, 3, True),     # 64 rows: GQA decode kernel, fixed splits
    (3, 48, 8, 8, 900, 2, False),     # 48 rows, non-causal block
    (1, 16, 1, 8, 1000, 4, True),     # 128 rows: 128-row kernel
])
def test_splitkv_then_merge_matches_oracle(B, Hq, Hkv, nq, L, splits, causal):
    wl = synth.Workload("t", "decode", B=B, Hq=Hq, Hkv=Hkv, Sq=nq, Lk=L, seed=B * 7 + Hq + nq, k_outliers=4,
                        q_outliers=True, outlier_mult=16.0, len_range=(L // 4, L))
    gen = wl.generate()
    qp, kp, vp, sl = quantize_on_gpu(gen)
    max_len = int(gen["seqlens"].max())
    ws = torch.empty((qk.decode_workspace_bytes(B, Hq, nq, splits),), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, nq, Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, nq), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    L_ = _lib.lib()
    rc = L_.qk4v8_attention_decode_splitkv(
        qp.codes.data_ptr(), qp.scales.data_ptr(), B, Hq, nq, qp.cap, kp.codes.data_ptr(), kp.scales.data_ptr(),
        vp.codes.data_ptr(), vp.scales.data_ptr(), Hkv, kp.cap, sl.data_ptr(), max_len, int(causal),
        ctypes.c_float(0.0), splits, ws.data_ptr(), ws.numel(), status.data_ptr(), stream)
    assert rc == 0, L_.qk4v8_last_error()
    rc = L_.qk4v8_decode_merge(ws.data_ptr(), ws.numel(), B, Hq, nq, splits, out.data_ptr(), lse.data_ptr(), stream)
    assert rc == 0, L_.qk4v8_last_error()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    (ref, rlse), _ = oracle_attention_from(gen, causal)
    assert_close(out, ref, f"splitkv+merge Hq={Hq} Hkv={Hkv} nq={nq}")
    got_lse = np.transpose(lse.cpu().numpy(), (0, 2, 1))
    fin = np.isfinite(rlse)
    assert np.array_equal(np.isfinite(got_lse), fin)
    assert np.abs(got_lse[fin] - rlse[fin]).max() < 1e-2
    rows = (Hq // Hkv) * nq
    if rows < 33 or rows > 64:
        # qk4v8_attention_decode with these splits runs the same split kernel and the same merge.
        one = qk.attention_decode(qp, kp, vp, sl, max_seqlen=max_len, causal_in_block=causal, num_splits=splits)
        torch.cuda.synchronize()
        assert torch.equal(one, out)


def test_merge_rejects_a_small_workspace():
    ws = torch.empty((1024,), dtype=torch.uint8, device="cuda")
    out = torch.empty((2, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    rc = _lib.lib().qk4v8_decode_merge(ws.data_ptr(), ws.numel(), 2, 8, 1, 4, out.data_ptr(), None,
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == 1
    assert b"workspace" in _lib.lib().qk4v8_last_error()
