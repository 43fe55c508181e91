"""Helpers shared by the GPU parity tests (test code only)."""
import numpy as np
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import oracle
from layouts import qk_scales_logical, unpack_e2m1, v_codes_logical, v_scales_logical

MAX_ABS_TOL = 3e-2   # attention output vs the fp64 oracle, unit-variance inputs
MEAN_ABS_TOL = 3e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16 numpy) -> CUDA bf16 tensor of the same shape."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def quantize_on_gpu(gen: dict, q_cap=None, kv_cap=None, nq_decode=False):
    q, k, v = to_dev(gen["q"]), to_dev(gen["k"]), to_dev(gen["v"])
    sl = torch.from_numpy(gen["seqlens"].astype(np.int32)).cuda()
    qp = qk.quantize_qk(q, cap=q_cap)
    kp = qk.quantize_qk(k, cap=kv_cap, seqlens=sl)
    vp = qk.quantize_v(v, cap=kv_cap, seqlens=sl)
    return qp, kp, vp, sl


def packed_to_logical(qp, kp, vp, Tq, Tk):
    """Library packed tensors -> oracle layout (codes one per byte)."""
    qc = unpack_e2m1(qp.codes.cpu().numpy()[:, :, :Tq])
    qs = qk_scales_logical(qp.scales.cpu().numpy(), Tq)
    kc = unpack_e2m1(kp.codes.cpu().numpy()[:, :, :Tk])
    ks = qk_scales_logical(kp.scales.cpu().numpy(), Tk)
    vc = v_codes_logical(vp.codes.cpu().numpy())[:, :, :, :Tk]
    vs = v_scales_logical(vp.scales.cpu().numpy(), Tk)
    return dict(qc=qc, qs=qs, kc=kc, ks=ks, vc=vc, vs=vs)


def err_stats(out: torch.Tensor, ref: np.ndarray):
    o = out.float().cpu().numpy().astype(np.float64)
    d = np.abs(o - ref)
    return float(d.max()), float(d.mean()), bool(np.isfinite(o).all())


def assert_close(out, ref, what=""):
    mx, mean, finite = err_stats(out, ref)
    assert finite, f"{what}: non-finite output"
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, f"{what}: max-abs {mx:.4g} mean-abs {mean:.4g}"
    return mx, mean


def oracle_attention_from(gen, causal, scale=None, sel=None):
    oz = oracle.quantize_workload(gen)
    return oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], gen["seqlens"],
                            causal=causal, scale=scale, sel=sel), oz
