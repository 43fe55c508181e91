"""ctypes loader for libqk4v8.so: one Python function per C entry point.

No fallback exists. If the shared library is missing or fails to load, every
call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqk4v8.so")

_lib = None

# Every exported entry point, with ctypes signatures (argtypes, restype).
_vp, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "qk4v8_status_string": ([_i32], ctypes.c_char_p),
    "qk4v8_last_error": ([], ctypes.c_char_p),
    "qk4v8_device_supported": ([_i32], _i32),
    "qk4v8_mxfp4_codes_bytes": ([_i32, _i32, _i32], _sz),
    "qk4v8_mxfp8_codes_bytes": ([_i32, _i32, _i32], _sz),
    "qk4v8_scales_bytes": ([_i32, _i32, _i32], _sz),
    "qk4v8_quantize_qk": ([_vp, _i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp], _i32),
    "qk4v8_quantize_qk_hadamard": ([_vp, _i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp], _i32),
    "qk4v8_quantize_v": ([_vp, _i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp], _i32),
    "qk4v8_quantize": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _i32, _i32,
                        _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_attention_prefill": ([_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                 _vp, _i32, _f32, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_decode_workspace_bytes": ([_i32, _i32, _i32, _i32], _sz),
    "qk4v8_decode_default_splits": ([_i32, _i32, _i32, _i32, _i32], _i32),
    "qk4v8_attention_decode": ([_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32,
                                _i32, _f32, _i32, _vp, _sz, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_attention_decode_splitkv": ([_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _vp,
                                        _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp], _i32),
    "qk4v8_decode_merge": ([_vp, _sz, _i32, _i32, _i32, _i32, _vp, _vp, _vp], _i32),
    "qk4v8_attention_decode_noalloc": ([_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _vp,
                                        _i32, _i32, _f32, _i32, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_attention_decode_window": ([_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _vp,
                                       _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_attention_decode_bf16_window": ([_vp, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i32,
                                            _vp, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_decode_default_splits_window": ([_i32, _i32, _i32, _i32, _i32, _i32], _i32),
    "qk4v8_decode_plan_splits": ([_i32, _i32, _i32, _i32, _vp, _i32], _i32),
    "qk4v8_mxfp4v_codes_bytes": ([_i32, _i32, _i32], _sz),
    "qk4v8_quantize_v4": ([_vp, _i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp], _i32),
    "qk4v8_attention_decode_v4": ([_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _vp,
                                   _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_attention_decode_bf16_v4": ([_vp, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i32,
                                        _vp, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_kv_tail_bytes": ([_i32, _i32], _sz),
    "qk4v8_kv_append": ([_vp, _vp, _i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _i32, _i32,
                         _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp], _i32),
    "qk4v8_attention_decode_paged": ([_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32,
                                      _vp, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_attention_decode_bf16_paged": ([_vp, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i32,
                                           _vp, _i32, _vp, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp, _vp,
                                           _vp], _i32),
    "qk4v8_decode_bf16_workspace_bytes": ([_i32, _i32, _i32, _i32, _i32], _sz),
    "qk4v8_attention_decode_bf16": ([_vp, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i32, _vp,
                                     _i32, _i32, _f32, _i32, _vp, _sz, _vp, _vp, _vp, _vp], _i32),
    "qk4v8_test_set_stall": ([_i32], None),
    "qk4v8_test_set_dump_scores": ([_vp], None),
    "qk4v8_test_set_force_swap_ab": ([_i32], None),
    "qk4v8_test_prefill_stage_qk": ([_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _vp, _i32, _f32,
                                     _vp, _vp, _vp], _i32),
    "qk4v8_test_mma_peak": ([_i32, _i32, _i32, _vp, _vp], _i32),
}


def lib():
    """The loaded library; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m bit_quantized_attention_qk4v8_b200.build` "
                "(there is no fallback implementation)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (argtypes, restype) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = argtypes
            fn.restype = restype
        _lib = handle
    return _lib


class QK4V8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        text = lib().qk4v8_last_error().decode(errors="replace")
        what = lib().qk4v8_status_string(status).decode()
        super().__init__(f"{where}: {what} ({status}): {text}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != 0:
        raise QK4V8Error(status, where)
