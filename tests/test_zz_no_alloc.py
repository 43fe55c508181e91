"""qk4v8_attention_decode_noalloc: decode for callers that cannot allocate.

Some callers may not call cudaMalloc. Examples are a plug-in inside a host
application that owns all device memory, and a latency-critical loop that
cannot take cudaMalloc's implicit synchronisation. This entry point gives them
decode with the split scratch held in a fixed device array inside the library.
The test calls it through the C ABI twice in a row, on different problems. Each
result must match qk4v8_attention_decode (caller workspace) within the
attention tolerance of the other tests. It also checks that an oversized
request is refused with a clear error.

This file is collected last on purpose and does not depend on any other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import synth
from bit_quantized_attention_qk4v8_b200 import _lib

pytestmark = pytest.mark.gpu

MAX_ABS_TOL = 3e-2
MEAN_ABS_TOL = 3e-3


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _problem(B, Hq, Hkv, nq, L, seed):
    wl = synth.Workload("noalloc", "decode", B=B, Hq=Hq, Hkv=Hkv, Sq=nq, Lk=L, seed=seed, k_outliers=4,
                        q_outliers=True, outlier_mult=16.0, len_range=(L // 3, L))
    gen = wl.generate()
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    qp = qk.quantize_qk(_dev(gen["q"]))
    kp = qk.quantize_qk(_dev(gen["k"]), seqlens=sl)
    vp = qk.quantize_v(_dev(gen["v"]), seqlens=sl)
    return qp, kp, vp, sl, int(gen["seqlens"].max())


def _noalloc(qp, kp, vp, sl, max_len, splits):
    out = torch.empty((qp.B, qp.length, qp.H, 128), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = _lib.lib().qk4v8_attention_decode_noalloc(
        qp.codes.data_ptr(), qp.scales.data_ptr(), qp.B, qp.H, qp.length, qp.cap,
        kp.codes.data_ptr(), kp.scales.data_ptr(), vp.codes.data_ptr(), vp.scales.data_ptr(), kp.H, kp.cap,
        sl.data_ptr(), max_len, 1, ctypes.c_float(0.0), splits, out.data_ptr(), None, status.data_ptr(), stream)
    assert rc == 0, _lib.lib().qk4v8_last_error()
    return out, status


def test_noalloc_decode_matches_workspace_decode_twice():
    cases = [dict(B=3, Hq=16, Hkv=4, nq=2, L=1500, seed=31, splits=3),
             dict(B=2, Hq=32, Hkv=8, nq=1, L=700, seed=32, splits=0)]
    for c in cases:
        qp, kp, vp, sl, max_len = _problem(c["B"], c["Hq"], c["Hkv"], c["nq"], c["L"], c["seed"])
        ref = qk.attention_decode(qp, kp, vp, sl, max_seqlen=max_len, num_splits=c["splits"])
        out, status = _noalloc(qp, kp, vp, sl, max_len, c["splits"])
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        d = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert d.max().item() <= MAX_ABS_TOL and d.mean().item() <= MEAN_ABS_TOL, (d.max().item(), d.mean().item())


def test_noalloc_rejects_oversized_scratch():
    qp, kp, vp, sl, max_len = _problem(2, 64, 8, 8, 600, 33)
    stream = torch.cuda.current_stream().cuda_stream
    out = torch.empty((qp.B, qp.length, qp.H, 128), dtype=torch.bfloat16, device="cuda")
    # 2*64*8 rows x 100 splits x 516 bytes is well beyond the fixed array.
    rc = _lib.lib().qk4v8_attention_decode_noalloc(
        qp.codes.data_ptr(), qp.scales.data_ptr(), qp.B, qp.H, qp.length, qp.cap,
        kp.codes.data_ptr(), kp.scales.data_ptr(), vp.codes.data_ptr(), vp.scales.data_ptr(), kp.H, kp.cap,
        sl.data_ptr(), max_len, 1, ctypes.c_float(0.0), 100, out.data_ptr(), None, None, stream)
    assert rc == 1
    assert b"exceeds the fixed" in _lib.lib().qk4v8_last_error()


def test_noalloc_gqa_kernel_after_other_contents():
    """33..64 query rows per KV head run on the GQA decode kernel, which keeps
    per-sequence piece counts in the scratch. A different call first leaves
    its own partials in the shared array; then two GQA problems in a row (splits
    >= 2, and the library's default) must still match qk4v8_attention_decode."""
    qp, kp, vp, sl, max_len = _problem(3, 16, 4, 2, 1500, 41)
    _noalloc(qp, kp, vp, sl, max_len, 4)          # fills the array with swap-AB partials
    torch.cuda.synchronize()
    for B, Hq, Hkv, nq, L, seed, splits in [(2, 64, 8, 8, 1200, 42, 3), (3, 48, 8, 8, 2000, 43, 0),
                                            (2, 64, 8, 8, 900, 44, 2)]:
        qp, kp, vp, sl, max_len = _problem(B, Hq, Hkv, nq, L, seed)
        ref = qk.attention_decode(qp, kp, vp, sl, max_seqlen=max_len, num_splits=splits)
        out, status = _noalloc(qp, kp, vp, sl, max_len, splits)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        d = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert d.max().item() <= MAX_ABS_TOL and d.mean().item() <= MEAN_ABS_TOL, (d.max().item(), d.mean().item())


def test_noalloc_single_split_needs_no_scratch():
    """One split with up to 64 rows writes the output directly: no size limit applies."""
    qp, kp, vp, sl, max_len = _problem(2, 32, 8, 1, 800, 45)
    ref = qk.attention_decode(qp, kp, vp, sl, max_seqlen=max_len, num_splits=1)
    out, status = _noalloc(qp, kp, vp, sl, max_len, 1)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out, ref)
