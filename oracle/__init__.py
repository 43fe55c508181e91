"""CPU oracle for QK4V8 attention: test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package. The library
(the CUDA path behind the C ABI) never does, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64). This module compiles it,
loads it with ctypes, and rearranges numpy arrays into the row order the C
functions take. The rearranging is plain indexing; it does no quantization or
attention arithmetic itself.

Tensor conventions (all numpy):
  bf16 inputs      uint16 bit patterns, [B, T, H, d]
  MXFP4 (Q, K)     codes uint8 [B, H, T, d] (one E2M1 code per byte),
                   scales uint8 [B, H, T, d/32] (E8M0)
  MXFP8 (V)        codes uint8 [B, Hkv, d, T] (E4M3),
                   scales uint8 [B, Hkv, d, ceil(T/32)] (E8M0), groups along T
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

E2M1 = 0
E4M3 = 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_decode.argtypes = [i32, i32]
        lib.oracle_decode.restype = ctypes.c_double
        lib.oracle_encode.argtypes = [i32, ctypes.c_double]
        lib.oracle_encode.restype = i32
        lib.oracle_shared_exponent.argtypes = [i32, ctypes.c_double]
        lib.oracle_shared_exponent.restype = i32
        lib.oracle_quantize_rows.argtypes = [vp, i64, i64, vp, i32, vp, vp]
        lib.oracle_quantize_rows.restype = i32
        lib.oracle_pack_e2m1.argtypes = [vp, i64, vp]
        lib.oracle_pack_e2m1.restype = i32
        lib.oracle_dequantize_rows.argtypes = [vp, vp, i64, i64, i32, vp]
        lib.oracle_dequantize_rows.restype = i32
        lib.oracle_attention.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                         ctypes.c_double, vp, i64, vp, vp]
        lib.oracle_attention.restype = i32
        lib.oracle_attention_window.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                                i32, ctypes.c_double, vp, i64, vp, vp]
        lib.oracle_attention_window.restype = i32
        lib.oracle_hadamard_rows.argtypes = [vp, i64, vp]
        lib.oracle_hadamard_rows.restype = i32
        lib.oracle_quantize_rows_f32.argtypes = [vp, i64, i64, vp, i32, vp, vp]
        lib.oracle_quantize_rows_f32.restype = i32
        lib.oracle_attention_ref.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                             ctypes.c_double, vp, i64, vp, vp]
        lib.oracle_attention_ref.restype = i32
        lib.oracle_num_threads.restype = i32
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def decode(fmt: int, code: int) -> float:
    return float(_load().oracle_decode(fmt, int(code)))


def encode(fmt: int, y: float) -> int:
    return int(_load().oracle_encode(fmt, float(y)))


def shared_exponent(fmt: int, amax: float) -> int:
    return int(_load().oracle_shared_exponent(fmt, float(amax)))


def quantize_rows(x_bits: np.ndarray, fmt: int, valid=None):
    """Quantize the last axis of `x_bits` (bf16 bits) in groups of 32."""
    lib = _load()
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n_cols = x.shape[-1]
    n_rows = x.size // n_cols
    ng = (n_cols + 31) // 32
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty(x.shape[:-1] + (ng,), dtype=np.uint8)
    vv = None
    if valid is not None:
        vv = np.ascontiguousarray(np.broadcast_to(valid, x.shape[:-1]), dtype=np.int32)
    rc = lib.oracle_quantize_rows(x.ctypes.data, n_rows, n_cols, vv.ctypes.data if vv is not None else None,
                                  fmt, codes.ctypes.data, scales.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle_quantize_rows failed")
    return codes, scales


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, fmt: int) -> np.ndarray:
    lib = _load()
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    n_cols = c.shape[-1]
    out = np.empty(c.shape, dtype=np.float64)
    lib.oracle_dequantize_rows(c.ctypes.data, s.ctypes.data, c.size // n_cols, n_cols, fmt, out.ctypes.data)
    return out


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    lib = _load()
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] // 2,), dtype=np.uint8)
    if lib.oracle_pack_e2m1(c.ctypes.data, c.size, out.ctypes.data) != 0:
        raise RuntimeError("odd element count")
    return out


def quantize_qk(x_bits: np.ndarray):
    """MXFP4 quantization of Q or K given as bf16 bits [B, T, H, d].

    Returns codes [B, H, T, d] and scales [B, H, T, d/32].
    """
    xt = np.ascontiguousarray(np.transpose(x_bits, (0, 2, 1, 3)))
    return quantize_rows(xt, E2M1)


def quantize_v(v_bits: np.ndarray, seqlens=None, fmt: int = E4M3):
    """MXFP8-E4M3 quantization of V given as bf16 bits [B, T, Hkv, d] (fmt=E2M1:
    MXFP4, the QK4V4 comparison point).

    Groups of 32 run along T. Returns codes [B, Hkv, d, T] and scales
    [B, Hkv, d, ceil(T/32)]; tokens at or past seqlens[b] are padding.
    """
    B, T, H, d = v_bits.shape
    vt = np.ascontiguousarray(np.transpose(v_bits, (0, 2, 3, 1)))
    valid = None
    if seqlens is not None:
        valid = np.broadcast_to(np.asarray(seqlens, dtype=np.int32)[:, None, None], (B, H, d))
    return quantize_rows(vt, fmt, valid)


def attention(qc, qs, kc, ks, vc, vs, seqlens=None, causal=True, scale=None, sel=None, window=0, v_fmt=E4M3):
    """fp64 attention over the dequantized MX tensors.

    qc/qs [B,Hq,Sq,d]/[B,Hq,Sq,d/32]; kc/ks [B,Hkv,Lk,d]/[B,Hkv,Lk,d/32];
    vc/vs [B,Hkv,d,Lk]/[B,Hkv,d,ceil(Lk/32)].
    sel: int32 [n,3] rows (b, h_q, i) or None for all rows.
    window > 0: each row sees only the last `window` keys before the query
    block and the block itself (the C function's visible_keys rule).
    v_fmt: element format of V's codes (E4M3, or E2M1 for QK4V4).
    Returns (out, lse): out [B,Sq,Hq,d] and lse [B,Sq,Hq] when sel is None,
    else out [n,d] and lse [n].
    """
    lib = _load()
    B, Hq, Sq, d = qc.shape
    Hkv, Lk = kc.shape[1], kc.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    arrs = [np.ascontiguousarray(a, dtype=np.uint8) for a in (qc, qs, kc, ks, vc, vs)]
    sl = None if seqlens is None else np.ascontiguousarray(seqlens, dtype=np.int32)
    n, selp, sela = _selection(sel, B * Sq * Hq)
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = lib.oracle_attention_window(*[a.ctypes.data for a in arrs], sl.ctypes.data if sl is not None else None,
                                     B, Hq, Hkv, Sq, Lk, d, int(bool(causal)), int(window), int(v_fmt),
                                     float(scale), selp, n,
                                     out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_attention_window failed ({rc})")
    if sel is None:
        return out.reshape(B, Sq, Hq, d), lse.reshape(B, Sq, Hq)
    return out, lse


def _selection(sel, n_all):
    if sel is None:
        return n_all, None, None
    sela = np.ascontiguousarray(sel, dtype=np.int32).reshape(-1, 3)
    return sela.shape[0], sela.ctypes.data, sela


def attention_ref(q, k, v, seqlens=None, causal=True, scale=None, sel=None, window=0):
    """fp64 softmax attention over UNQUANTIZED inputs (the context reference).

    q [B,Sq,Hq,d], k and v [B,Lk,Hkv,d]: float32 arrays, or uint16 bf16 bit
    patterns (converted exactly). Masking as for `attention`. Returns (out,
    lse) shaped like `attention`'s.
    """
    lib = _load()
    q, k, v = (_as_f32(t) for t in (q, k, v))
    B, Sq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    sl = None if seqlens is None else np.ascontiguousarray(seqlens, dtype=np.int32)
    n, selp, sela = _selection(sel, B * Sq * Hq)
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = lib.oracle_attention_ref(q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                  sl.ctypes.data if sl is not None else None, B, Hq, Hkv, Sq, Lk, d,
                                  int(bool(causal)), int(window), float(scale), selp, n, out.ctypes.data,
                                  lse.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_attention_ref failed ({rc})")
    if sel is None:
        return out.reshape(B, Sq, Hq, d), lse.reshape(B, Sq, Hq)
    return out, lse


def _as_f32(t):
    """float32 array as is; uint16 bf16 bit patterns widened to float32 (a bit shift, exact)."""
    t = np.asarray(t)
    if t.dtype == np.uint16:
        return np.ascontiguousarray((t.astype(np.uint32) << 16).view(np.float32))
    return np.ascontiguousarray(t, dtype=np.float32)


def hadamard_rows(x_bits: np.ndarray) -> np.ndarray:
    """Rotation of 128-channel rows (bf16 bits [..., 128]) by H/sqrt(128), in fp32 (oracle.c)."""
    lib = _load()
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if x.shape[-1] != 128:
        raise ValueError("rows of 128 channels")
    y = np.empty(x.shape, dtype=np.float32)
    if lib.oracle_hadamard_rows(x.ctypes.data, x.size // 128, y.ctypes.data) != 0:
        raise RuntimeError("oracle_hadamard_rows failed")
    return y


def quantize_rows_f32(x: np.ndarray, fmt: int, valid=None):
    """quantize_rows for float32 values (last axis, groups of 32)."""
    lib = _load()
    xf = np.ascontiguousarray(x, dtype=np.float32)
    n_cols = xf.shape[-1]
    ng = (n_cols + 31) // 32
    codes = np.empty(xf.shape, dtype=np.uint8)
    scales = np.empty(xf.shape[:-1] + (ng,), dtype=np.uint8)
    vv = None
    if valid is not None:
        vv = np.ascontiguousarray(np.broadcast_to(valid, xf.shape[:-1]), dtype=np.int32)
    rc = lib.oracle_quantize_rows_f32(xf.ctypes.data, xf.size // n_cols, n_cols,
                                      vv.ctypes.data if vv is not None else None, fmt, codes.ctypes.data,
                                      scales.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle_quantize_rows_f32 failed")
    return codes, scales


def quantize_qk_hadamard(x_bits: np.ndarray, seqlens=None):
    """MXFP4 quantization of Hadamard-rotated Q or K, bf16 bits [B, T, H, d].

    Each (token, head) row is rotated by H/sqrt(128) in fp32 and then
    quantized like quantize_qk. Tokens at or past seqlens[b] (when given) get
    zero codes and scales. Returns codes [B, H, T, d] and scales [B, H, T, d/32].
    """
    xt = np.ascontiguousarray(np.transpose(x_bits, (0, 2, 1, 3)))
    y = hadamard_rows(xt)
    valid = None
    if seqlens is not None:
        B, H, T, d = xt.shape
        lens = np.asarray(seqlens, dtype=np.int64)
        valid = np.where(np.arange(T)[None, None, :] < lens[:, None, None], d, 0).astype(np.int32)
        valid = np.broadcast_to(valid, (B, H, T))
    return quantize_rows_f32(y, E2M1, valid)


def quantize_workload(gen: dict, v_fmt: int = E4M3):
    """Oracle quantization of a generated workload dict (q, k, v, seqlens)."""
    qc, qs = quantize_qk(gen["q"])
    kc, ks = quantize_qk(gen["k"])
    vc, vs = quantize_v(gen["v"], gen["seqlens"], v_fmt)
    return dict(qc=qc, qs=qs, kc=kc, ks=ks, vc=vc, vs=vs)
