"""QK4V8 mixed-precision attention for B200 (sm_100a).

This is the Python binding of libqk4v8.so. It marshals arguments only: torch
provides device memory and the current stream, and every step of the
computation runs in the library's CUDA kernels. Function names follow the C
entry points in include/qk4v8.h.

Method (MpFA QK4V8 article, mhpn.cn):
  - Q and K are quantized to MXFP4 and V to MXFP8-E4M3, with one E8M0 scale
    per 32 values computed online.
  - Attention then runs tile by tile with an FP32 online softmax, on
    block-scaled tcgen05 tensor-core MMAs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch

from ._lib import QK4V8Error, check, lib

__all__ = [
    "MXFP4", "MXFP4V", "MXFP8V", "PagedKV", "QK4V8Error", "lib", "round_cap",
    "quantize_qk", "quantize_v", "quantize", "attention_prefill", "attention_decode",
    "decode_workspace_bytes", "decode_default_splits", "decode_plan_splits", "attention_decode_splitkv",
    "decode_merge",
    "attention_decode_bf16", "decode_bf16_workspace_bytes",
    "paged_kv", "kv_append", "attention_decode_paged", "attention_decode_bf16_paged", "quantize_v4",
]

D = 128


def round_cap(n: int) -> int:
    """Smallest multiple of 128 that holds n tokens (at least 128)."""
    return max(128, (int(n) + 127) // 128 * 128)


@dataclass
class MXFP4:
    """Packed MXFP4 tensor (Q or K): codes uint8 [B][H][cap][64], scales uint8 [B][H][cap/128][512]."""
    codes: torch.Tensor
    scales: torch.Tensor
    B: int
    H: int
    cap: int
    length: int


@dataclass
class MXFP4V:
    """Packed MXFP4 V (the QK4V4 comparison point): codes uint8 [B][H][cap/128][128][64]
    (128-token blocks of channel rows, two tokens per byte), scales uint8 [B][H][cap/128][512]."""
    codes: torch.Tensor
    scales: torch.Tensor
    B: int
    H: int
    cap: int
    length: int


@dataclass
class MXFP8V:
    """Packed MXFP8-E4M3 V: codes uint8 [B][H][cap/128][128][128] (128-token blocks of
    channel rows), scales uint8 [B][H][cap/128][512]."""
    codes: torch.Tensor
    scales: torch.Tensor
    B: int
    H: int
    cap: int
    length: int


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_bf16(x: torch.Tensor, name: str):
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 4 or x.shape[-1] != D or x.stride(-1) != 1:
        raise ValueError(f"{name} must be a CUDA bf16 tensor [B, T, H, 128] with unit channel stride")


def _seqlens(seqlens, B, device):
    if seqlens is None:
        return None
    if not torch.is_tensor(seqlens):
        seqlens = torch.tensor(seqlens, dtype=torch.int32)
    seqlens = seqlens.to(device=device, dtype=torch.int32).contiguous()
    if seqlens.numel() != B:
        raise ValueError("seqlens must have B entries")
    return seqlens


def quantize_qk(x: torch.Tensor, cap: Optional[int] = None, seqlens=None, out: Optional[MXFP4] = None,
                hadamard: bool = False) -> MXFP4:
    """MXFP4-quantize Q or K ([B, T, H, 128] bf16) into the packed layout.

    hadamard=True rotates each row by H/sqrt(128) first (qk4v8_quantize_qk_hadamard);
    rotate both Q and K, or neither."""
    _check_bf16(x, "x")
    B, T, H, _ = x.shape
    cap = round_cap(T) if cap is None else int(cap)
    sl = _seqlens(seqlens, B, x.device)
    if out is None:
        out = MXFP4(torch.empty((B, H, cap, 64), dtype=torch.uint8, device=x.device),
                    torch.empty((B, H, cap // 128, 512), dtype=torch.uint8, device=x.device), B, H, cap, T)
    fn, name = ((lib().qk4v8_quantize_qk_hadamard, "qk4v8_quantize_qk_hadamard") if hadamard
                else (lib().qk4v8_quantize_qk, "qk4v8_quantize_qk"))
    check(fn(x.data_ptr(), B, T, H, D, x.stride(0), x.stride(1), x.stride(2), _ptr(sl), cap,
             out.codes.data_ptr(), out.scales.data_ptr(), _stream(x.device)), name)
    out.length = T
    return out


def quantize_v(v: torch.Tensor, cap: Optional[int] = None, seqlens=None, out: Optional[MXFP8V] = None) -> MXFP8V:
    """MXFP8-E4M3-quantize V ([B, T, H, 128] bf16), groups of 32 along T."""
    _check_bf16(v, "v")
    B, T, H, _ = v.shape
    cap = round_cap(T) if cap is None else int(cap)
    sl = _seqlens(seqlens, B, v.device)
    if out is None:
        out = MXFP8V(torch.empty((B, H, cap // 128, D, 128), dtype=torch.uint8, device=v.device),
                     torch.empty((B, H, cap // 128, 512), dtype=torch.uint8, device=v.device), B, H, cap, T)
    check(lib().qk4v8_quantize_v(v.data_ptr(), B, T, H, D, v.stride(0), v.stride(1), v.stride(2), _ptr(sl), cap,
                                 out.codes.data_ptr(), out.scales.data_ptr(), _stream(v.device)), "qk4v8_quantize_v")
    out.length = T
    return out


def quantize_v4(v: torch.Tensor, cap: Optional[int] = None, seqlens=None, out: Optional[MXFP4V] = None) -> MXFP4V:
    """MXFP4-quantize V ([B, T, H, 128] bf16), groups of 32 along T (qk4v8_quantize_v4, QK4V4)."""
    _check_bf16(v, "v")
    B, T, H, _ = v.shape
    cap = round_cap(T) if cap is None else int(cap)
    sl = _seqlens(seqlens, B, v.device)
    if out is None:
        out = MXFP4V(torch.empty((B, H, cap // 128, D, 64), dtype=torch.uint8, device=v.device),
                     torch.empty((B, H, cap // 128, 512), dtype=torch.uint8, device=v.device), B, H, cap, T)
    check(lib().qk4v8_quantize_v4(v.data_ptr(), B, T, H, D, v.stride(0), v.stride(1), v.stride(2), _ptr(sl), cap,
                                  out.codes.data_ptr(), out.scales.data_ptr(), _stream(v.device)), "qk4v8_quantize_v4")
    out.length = T
    return out


def quantize(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seqlens_k=None, q_cap=None, kv_cap=None,
             hadamard: bool = False):
    """Quantize contiguous Q [B,Sq,Hq,128], K and V [B,Sk,Hkv,128] in one library call.

    hadamard=True quantizes Q and K after their Hadamard rotation (three launches:
    qk4v8_quantize_qk_hadamard for Q and K, qk4v8_quantize_v for V)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous for qk4v8_quantize")
    B, Sq, Hq, _ = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    q_cap = round_cap(Sq) if q_cap is None else int(q_cap)
    kv_cap = round_cap(Sk) if kv_cap is None else int(kv_cap)
    dev = q.device
    sl = _seqlens(seqlens_k, B, dev)
    if hadamard:
        qp = quantize_qk(q, cap=q_cap, hadamard=True)
        kp = quantize_qk(k, cap=kv_cap, seqlens=sl, hadamard=True)
        vp = quantize_v(v, cap=kv_cap, seqlens=sl)
        return qp, kp, vp
    qp = MXFP4(torch.empty((B, Hq, q_cap, 64), dtype=torch.uint8, device=dev),
               torch.empty((B, Hq, q_cap // 128, 512), dtype=torch.uint8, device=dev), B, Hq, q_cap, Sq)
    kp = MXFP4(torch.empty((B, Hkv, kv_cap, 64), dtype=torch.uint8, device=dev),
               torch.empty((B, Hkv, kv_cap // 128, 512), dtype=torch.uint8, device=dev), B, Hkv, kv_cap, Sk)
    vp = MXFP8V(torch.empty((B, Hkv, kv_cap // 128, D, 128), dtype=torch.uint8, device=dev),
                torch.empty((B, Hkv, kv_cap // 128, 512), dtype=torch.uint8, device=dev), B, Hkv, kv_cap, Sk)
    check(lib().qk4v8_quantize(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Sq, Sk, Hq, Hkv, D, _ptr(sl), q_cap,
                               kv_cap, qp.codes.data_ptr(), qp.scales.data_ptr(), kp.codes.data_ptr(),
                               kp.scales.data_ptr(), vp.codes.data_ptr(), vp.scales.data_ptr(), _stream(dev)),
          "qk4v8_quantize")
    return qp, kp, vp


def attention_prefill(q: MXFP4, k: MXFP4, v: MXFP8V, seqlens_k=None, causal: bool = True,
                      softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] = None, return_lse: bool = False,
                      dev_status: Optional[torch.Tensor] = None):
    """QK4V8 prefill attention. Returns out bf16 [B, Sq, Hq, 128] (and lse [B, Hq, Sq])."""
    dev = q.codes.device
    B, Hq, Sq = q.B, q.H, q.length
    sl = _seqlens(seqlens_k, B, dev)
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
    check(lib().qk4v8_attention_prefill(q.codes.data_ptr(), q.scales.data_ptr(), B, Hq, Sq, q.cap,
                                        k.codes.data_ptr(), k.scales.data_ptr(), v.codes.data_ptr(),
                                        v.scales.data_ptr(), k.H, k.length, k.cap, _ptr(sl), int(bool(causal)),
                                        float(softmax_scale or 0.0), out.data_ptr(), _ptr(lse), _ptr(dev_status),
                                        _stream(dev)), "qk4v8_attention_prefill")
    return (out, lse) if return_lse else out


def decode_workspace_bytes(B: int, Hq: int, nq: int, num_splits: int) -> int:
    return int(lib().qk4v8_decode_workspace_bytes(B, Hq, nq, num_splits))


def decode_default_splits(B: int, Hq: int, Hkv: int, nq: int, max_seqlen: int, window: int = 0) -> int:
    if window:
        return int(lib().qk4v8_decode_default_splits_window(B, Hq, Hkv, nq, max_seqlen, int(window)))
    return int(lib().qk4v8_decode_default_splits(B, Hq, Hkv, nq, max_seqlen))


def decode_plan_splits(B: int, Hq: int, Hkv: int, nq: int, seqlens, window: int = 0) -> int:
    """Split count from the host-side sequence lengths (qk4v8_decode_plan_splits)."""
    import numpy as np
    lens = np.ascontiguousarray(np.asarray(seqlens if not torch.is_tensor(seqlens) else seqlens.cpu().numpy()),
                                dtype=np.int32)
    if lens.size != B:
        raise ValueError("seqlens must have B entries")
    return int(lib().qk4v8_decode_plan_splits(B, Hq, Hkv, nq, lens.ctypes.data, int(window)))


def attention_decode(q: MXFP4, k: MXFP4, v, seqlens_k, max_seqlen: Optional[int] = None,
                     causal_in_block: bool = True, softmax_scale: Optional[float] = None, num_splits: int = 0,
                     workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, return_lse: bool = False,
                     dev_status: Optional[torch.Tensor] = None, window: int = 0):
    """Split-KV decode / speculative verify over a packed cache. Returns out bf16 [B, nq, Hq, 128].

    window > 0: draft-block attention, each query row sees only the last `window`
    keys before the nq-token block and the block (qk4v8_attention_decode_window)."""
    dev = q.codes.device
    B, Hq, nq = q.B, q.H, q.length
    sl = _seqlens(seqlens_k, B, dev)
    if max_seqlen is None:
        max_seqlen = k.cap
    splits = num_splits if num_splits > 0 else decode_default_splits(B, Hq, k.H, nq, max_seqlen, window)
    need = decode_workspace_bytes(B, Hq, nq, splits)
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, nq, Hq, D), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, nq), dtype=torch.float32, device=dev)
    head = (q.codes.data_ptr(), q.scales.data_ptr(), B, Hq, nq, q.cap, k.codes.data_ptr(), k.scales.data_ptr(),
            v.codes.data_ptr(), v.scales.data_ptr(), k.H, k.cap, _ptr(sl), int(max_seqlen),
            int(bool(causal_in_block)))
    tail = (float(softmax_scale or 0.0), int(splits), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), out.data_ptr(), _ptr(lse), _ptr(dev_status), _stream(dev))
    if isinstance(v, MXFP4V):
        check(lib().qk4v8_attention_decode_v4(*head, int(window), *tail), "qk4v8_attention_decode_v4")
    elif window:
        check(lib().qk4v8_attention_decode_window(*head, int(window), *tail), "qk4v8_attention_decode_window")
    else:
        check(lib().qk4v8_attention_decode(*head, *tail), "qk4v8_attention_decode")
    return (out, lse) if return_lse else out


def decode_bf16_workspace_bytes(B: int, Hq: int, Hkv: int, nq: int, num_splits: int) -> int:
    return int(lib().qk4v8_decode_bf16_workspace_bytes(B, Hq, Hkv, nq, num_splits))


def attention_decode_bf16(q: torch.Tensor, k: MXFP4, v, seqlens_k, max_seqlen: Optional[int] = None,
                          causal_in_block: bool = True, softmax_scale: Optional[float] = None, num_splits: int = 0,
                          workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                          lse: Optional[torch.Tensor] = None, return_lse: bool = False,
                          dev_status: Optional[torch.Tensor] = None, window: int = 0):
    """Decode step from bf16 queries q [B, nq, Hq, 128]; the query is MXFP4-quantized inside the call.
    Returns out bf16 [B, nq, Hq, 128] (and lse [B, Hq, nq]). window as for attention_decode."""
    _check_bf16(q, "q")
    dev = q.device
    B, nq, Hq, _ = q.shape
    sl = _seqlens(seqlens_k, B, dev)
    if max_seqlen is None:
        max_seqlen = k.cap
    splits = num_splits if num_splits > 0 else decode_default_splits(B, Hq, k.H, nq, max_seqlen, window)
    need = decode_bf16_workspace_bytes(B, Hq, k.H, nq, splits)
    if workspace is None and need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, nq, Hq, D), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, nq), dtype=torch.float32, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    head = (q.data_ptr(), B, Hq, nq, q.stride(0), q.stride(1), q.stride(2), k.codes.data_ptr(), k.scales.data_ptr(),
            v.codes.data_ptr(), v.scales.data_ptr(), k.H, k.cap, _ptr(sl), int(max_seqlen),
            int(bool(causal_in_block)))
    tail = (float(softmax_scale or 0.0), int(splits), _ptr(workspace), ws_bytes, out.data_ptr(), _ptr(lse),
            _ptr(dev_status), _stream(dev))
    if isinstance(v, MXFP4V):
        check(lib().qk4v8_attention_decode_bf16_v4(*head, int(window), *tail), "qk4v8_attention_decode_bf16_v4")
    elif window:
        check(lib().qk4v8_attention_decode_bf16_window(*head, int(window), *tail), "qk4v8_attention_decode_bf16_window")
    else:
        check(lib().qk4v8_attention_decode_bf16(*head, *tail), "qk4v8_attention_decode_bf16")
    return (out, lse) if return_lse else out


def attention_decode_splitkv(q: MXFP4, k: MXFP4, v: MXFP8V, seqlens_k: torch.Tensor, max_seqlen: int,
                             num_splits: int, workspace: torch.Tensor, causal_in_block: bool = True,
                             softmax_scale: Optional[float] = None, dev_status: Optional[torch.Tensor] = None):
    """First decode stage: per-split partial (O, lse2) into `workspace` (num_splits must be > 0)."""
    dev = q.codes.device
    check(lib().qk4v8_attention_decode_splitkv(q.codes.data_ptr(), q.scales.data_ptr(), q.B, q.H, q.length, q.cap,
                                               k.codes.data_ptr(), k.scales.data_ptr(), v.codes.data_ptr(),
                                               v.scales.data_ptr(), k.H, k.cap, seqlens_k.data_ptr(),
                                               int(max_seqlen), int(bool(causal_in_block)),
                                               float(softmax_scale or 0.0), int(num_splits), workspace.data_ptr(),
                                               workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                               _stream(dev)), "qk4v8_attention_decode_splitkv")


def decode_merge(workspace: torch.Tensor, B: int, Hq: int, nq: int, num_splits: int, out: torch.Tensor,
                 lse: Optional[torch.Tensor] = None):
    """Second decode stage: merge the split partials into out bf16 [B, nq, Hq, 128]."""
    check(lib().qk4v8_decode_merge(workspace.data_ptr(), workspace.numel() * workspace.element_size(), B, Hq, nq,
                                   num_splits, out.data_ptr(), _ptr(lse), _stream(out.device)), "qk4v8_decode_merge")
    return out


def default_scale() -> float:
    return 1.0 / math.sqrt(D)


# ----------------------------------------------------------------------------------------------------------
# Measurement hooks (include/qk4v8_test.h): not part of the attention API.

def prefill_stage_qk(q: MXFP4, k: MXFP4, seqlens_k=None, causal: bool = True,
                     softmax_scale: Optional[float] = None, row_max: Optional[torch.Tensor] = None,
                     dev_status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The QK^T stage of the prefill kernel alone (same tile schedule, no exp / P / PV).

    Returns row_max float32 [B, Hq, Sq]: each query row's largest allowed score
    times softmax_scale * log2(e) (-inf for a row with no allowed key).
    """
    dev = q.codes.device
    B, Hq, Sq = q.B, q.H, q.length
    sl = _seqlens(seqlens_k, B, dev)
    if row_max is None:
        row_max = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
    check(lib().qk4v8_test_prefill_stage_qk(q.codes.data_ptr(), q.scales.data_ptr(), B, Hq, Sq, q.cap,
                                            k.codes.data_ptr(), k.scales.data_ptr(), k.H, k.length, k.cap, _ptr(sl),
                                            int(bool(causal)), float(softmax_scale or 0.0), row_max.data_ptr(),
                                            _ptr(dev_status), _stream(dev)), "qk4v8_test_prefill_stage_qk")
    return row_max


MMA_PEAK_SHAPES = {0: ("mxf4", 128, 128, 64), 1: ("mxf8f6f4", 128, 144, 32),
                   2: ("mxf8f6f4", 128, 256, 32), 3: ("mxf4", 128, 256, 64)}


def mma_peak_run(kind: int, ctas: int, iters: int, device=None, dev_status: Optional[torch.Tensor] = None) -> int:
    """Enqueue one tensor-pipe peak run; returns its FLOP count (2*M*N*K per instruction)."""
    dev = torch.device(device or "cuda")
    check(lib().qk4v8_test_mma_peak(int(kind), int(ctas), int(iters), _ptr(dev_status), _stream(dev)),
          "qk4v8_test_mma_peak")
    _, m, n, kk = MMA_PEAK_SHAPES[int(kind)]
    return 2 * m * n * kk * int(ctas) * int(iters)


# ----------------------------------------------------------------------------------------------------------
# Paged KV cache (include/qk4v8.h: qk4v8_kv_append, qk4v8_attention_decode_paged).

@dataclass
class PagedKV:
    """Packed KV cache in pools of 128-token pages, and the per-sequence state.

    k_codes uint8 [P, Hkv, 128, 64], k_scales uint8 [P, Hkv, 512],
    v_codes uint8 [P, Hkv, 128, 128], v_scales uint8 [P, Hkv, 512] (P pages);
    block_table int32 [B, max_pages]: page of each 128-token block of a sequence;
    seqlens int32 [B]: tokens held; v_tail bf16 [B, Hkv, 32, 128]: the open V
    group of each sequence and head, which every append reads and refreshes."""
    k_codes: torch.Tensor
    k_scales: torch.Tensor
    v_codes: torch.Tensor
    v_scales: torch.Tensor
    v_tail: torch.Tensor
    block_table: torch.Tensor
    seqlens: torch.Tensor
    hadamard_k: bool = False

    @property
    def num_pages(self) -> int:
        return self.k_codes.shape[0]

    @property
    def Hkv(self) -> int:
        return self.k_codes.shape[1]

    @property
    def B(self) -> int:
        return self.block_table.shape[0]

    @property
    def max_pages(self) -> int:
        return self.block_table.shape[1]


def paged_kv(B: int, Hkv: int, num_pages: int, block_table: torch.Tensor, device="cuda",
             hadamard_k: bool = False) -> PagedKV:
    """An empty paged cache (every sequence of length 0) over a new pool of num_pages pages.
    block_table: int32 [B, max_pages] page indices, owned by the caller's page allocator."""
    dev = torch.device(device)
    bt = block_table.to(device=dev, dtype=torch.int32).contiguous()
    if bt.dim() != 2 or bt.shape[0] != B:
        raise ValueError("block_table must be [B, max_pages]")
    u8 = torch.uint8
    return PagedKV(k_codes=torch.empty((num_pages, Hkv, 128, 64), dtype=u8, device=dev),
                   k_scales=torch.empty((num_pages, Hkv, 512), dtype=u8, device=dev),
                   v_codes=torch.empty((num_pages, Hkv, 128, 128), dtype=u8, device=dev),
                   v_scales=torch.empty((num_pages, Hkv, 512), dtype=u8, device=dev),
                   v_tail=torch.empty((B, Hkv, 32, 128), dtype=torch.bfloat16, device=dev),
                   block_table=bt, seqlens=torch.zeros((B,), dtype=torch.int32, device=dev), hadamard_k=hadamard_k)


def kv_append(cache: PagedKV, k_new: torch.Tensor, v_new: torch.Tensor, dev_status: Optional[torch.Tensor] = None):
    """Append k_new, v_new (bf16 [B, n_new, Hkv, 128], same strides) to every sequence
    (qk4v8_kv_append); cache.seqlens advances by n_new on the device."""
    _check_bf16(k_new, "k_new")
    _check_bf16(v_new, "v_new")
    if k_new.shape != v_new.shape or k_new.stride() != v_new.stride():
        raise ValueError("k_new and v_new must have the same shape and strides")
    B, n_new, Hkv, _ = k_new.shape
    check(lib().qk4v8_kv_append(k_new.data_ptr(), v_new.data_ptr(), B, n_new, Hkv, D, k_new.stride(0),
                                k_new.stride(1), k_new.stride(2), cache.seqlens.data_ptr(),
                                cache.seqlens.data_ptr(), cache.block_table.data_ptr(), cache.max_pages,
                                cache.num_pages, cache.k_codes.data_ptr(), cache.k_scales.data_ptr(),
                                cache.v_codes.data_ptr(), cache.v_scales.data_ptr(), cache.v_tail.data_ptr(),
                                int(cache.hadamard_k), _ptr(dev_status), _stream(k_new.device)), "qk4v8_kv_append")
    return cache


def _paged_call_args(cache: PagedKV):
    return (cache.k_codes.data_ptr(), cache.k_scales.data_ptr(), cache.v_codes.data_ptr(), cache.v_scales.data_ptr(),
            cache.Hkv, cache.num_pages, cache.block_table.data_ptr(), cache.max_pages, cache.seqlens.data_ptr())


def attention_decode_paged(q: MXFP4, cache: PagedKV, max_seqlen: int, causal_in_block: bool = True,
                           window: int = 0, softmax_scale: Optional[float] = None, num_splits: int = 0,
                           workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None, return_lse: bool = False,
                           dev_status: Optional[torch.Tensor] = None):
    """Decode / verify / draft-block attention over a paged cache (qk4v8_attention_decode_paged)."""
    dev = q.codes.device
    B, Hq, nq = q.B, q.H, q.length
    splits = num_splits if num_splits > 0 else decode_default_splits(B, Hq, cache.Hkv, nq, max_seqlen, window)
    if workspace is None:
        workspace = torch.empty((max(16, decode_workspace_bytes(B, Hq, nq, splits)),), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, nq, Hq, D), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, nq), dtype=torch.float32, device=dev)
    check(lib().qk4v8_attention_decode_paged(q.codes.data_ptr(), q.scales.data_ptr(), B, Hq, nq, q.cap,
                                             *_paged_call_args(cache), int(max_seqlen), int(bool(causal_in_block)),
                                             int(window), float(softmax_scale or 0.0), int(splits),
                                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                             out.data_ptr(), _ptr(lse), _ptr(dev_status), _stream(dev)),
          "qk4v8_attention_decode_paged")
    return (out, lse) if return_lse else out


def attention_decode_bf16_paged(q: torch.Tensor, cache: PagedKV, max_seqlen: int, causal_in_block: bool = True,
                                window: int = 0, softmax_scale: Optional[float] = None, num_splits: int = 0,
                                workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                                lse: Optional[torch.Tensor] = None, return_lse: bool = False,
                                dev_status: Optional[torch.Tensor] = None):
    """Decode step from bf16 queries q [B, nq, Hq, 128] over a paged cache (qk4v8_attention_decode_bf16_paged)."""
    _check_bf16(q, "q")
    dev = q.device
    B, nq, Hq, _ = q.shape
    splits = num_splits if num_splits > 0 else decode_default_splits(B, Hq, cache.Hkv, nq, max_seqlen, window)
    need = decode_bf16_workspace_bytes(B, Hq, cache.Hkv, nq, splits)
    if workspace is None and need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, nq, Hq, D), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, nq), dtype=torch.float32, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib().qk4v8_attention_decode_bf16_paged(q.data_ptr(), B, Hq, nq, q.stride(0), q.stride(1), q.stride(2),
                                                  *_paged_call_args(cache), int(max_seqlen),
                                                  int(bool(causal_in_block)), int(window),
                                                  float(softmax_scale or 0.0), int(splits), _ptr(workspace), ws_bytes,
                                                  out.data_ptr(), _ptr(lse), _ptr(dev_status), _stream(dev)),
          "qk4v8_attention_decode_bf16_paged")
    return (out, lse) if return_lse else out
