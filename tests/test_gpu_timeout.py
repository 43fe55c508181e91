"""Failure detection without a GPU fault: a pipeline wait that runs out.

The test hook withholds each attention launch's "Q tile ready" signal, so the
kernel's bounded waits expire after about a second. The kernel then writes
QK4V8_ERR_TIMEOUT to dev_status, unwinds, frees its tensor memory and
returns; the host reads the status, and the CUDA context stays usable for
the next (normal) launch.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import synth
from bit_quantized_attention_qk4v8_b200 import _lib
from gpu_util import quantize_on_gpu

pytestmark = pytest.mark.gpu

QK4V8_ERR_TIMEOUT = 4


def small_gen(B, Sq, Lk, Hq, Hkv, seed):
    wl = synth.Workload("t", "decode", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Lk=Lk, seed=seed)
    return wl.generate()


def stalled(fn):
    _lib.lib().qk4v8_test_set_stall(1)
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        _lib.lib().qk4v8_test_set_stall(0)


@pytest.mark.timeout(120)
def test_prefill_wait_times_out_and_context_survives():
    gen = small_gen(1, 256, 256, 2, 1, seed=5)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    ref = qk.attention_prefill(qp, kp, vp, seqlens_k=sl)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stalled(lambda: qk.attention_prefill(qp, kp, vp, seqlens_k=sl, dev_status=status))
    assert int(status.item()) == QK4V8_ERR_TIMEOUT
    # The context is usable and the next launch is correct.
    again = qk.attention_prefill(qp, kp, vp, seqlens_k=sl)
    torch.cuda.synchronize()
    assert torch.equal(again, ref)


@pytest.mark.timeout(120)
@pytest.mark.parametrize("Hq,nq", [(8, 1), (16, 8)])
def test_decode_wait_times_out_and_context_survives(Hq, nq):
    gen = small_gen(2, nq, 700, Hq, 2, seed=6)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    ref = qk.attention_decode(qp, kp, vp, sl, max_seqlen=700, num_splits=2)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stalled(lambda: qk.attention_decode(qp, kp, vp, sl, max_seqlen=700, num_splits=2, dev_status=status))
    assert int(status.item()) == QK4V8_ERR_TIMEOUT
    again = qk.attention_decode(qp, kp, vp, sl, max_seqlen=700, num_splits=2)
    torch.cuda.synchronize()
    assert torch.equal(again, ref)


@pytest.mark.timeout(60)
def test_status_stays_clear_on_normal_launches():
    gen = small_gen(1, 130, 300, 4, 2, seed=7)
    qp, kp, vp, sl = quantize_on_gpu(gen)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    qk.attention_prefill(qp, kp, vp, seqlens_k=sl, dev_status=status)
    qdec = qk.quantize_qk(torch.zeros((1, 1, 4, 128), dtype=torch.bfloat16, device="cuda"))
    qk.attention_decode(qdec, kp, vp, sl, max_seqlen=300, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
