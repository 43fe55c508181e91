"""Seeded synthetic inputs for the QK4V8 attention workloads.

This module only generates inputs: bf16 bit patterns of Q, K, V in
[B, T, H, D] order plus per-sequence KV lengths. It contains no quantization
or attention arithmetic. The CPU oracle and the CUDA path both read its output
unchanged.

The random numbers come from the counter-based generator in ``gen.c``. The
workload recipes (shapes, distributions, outlier channels, length mixes) are
the five workloads the MpFA QK4V8 article is benchmarked on here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

DIST_NORMAL = 0
DIST_STUDENT_T3 = 1

STREAM_Q, STREAM_K, STREAM_V, STREAM_PICK, STREAM_LENS = 0, 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile gen.c into libsynth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.synth_fill.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                   ctypes.c_int, ctypes.c_void_p, ctypes.c_uint16]
        lib.synth_fill.restype = ctypes.c_int
        lib.synth_pick_channels.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_pick_channels.restype = ctypes.c_int
        lib.synth_uniform_ints.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_uniform_ints.restype = ctypes.c_int
        lib.synth_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def fill(B, T, H, D, seed, stream, dist=DIST_NORMAL, chan_mult=None, t_valid=None, pad_bits=0):
    """bf16 bits [B, T, H, D] drawn from stream `stream` of `seed`."""
    lib = _load()
    out = np.empty((B, T, H, D), dtype=np.uint16)
    cm = None
    if chan_mult is not None:
        cm = np.ascontiguousarray(chan_mult, dtype=np.float32).reshape(H, D)
    tv = None
    if t_valid is not None:
        tv = np.ascontiguousarray(t_valid, dtype=np.int32)
    rc = lib.synth_fill(out.ctypes.data, B, T, H, D,
                        tv.ctypes.data if tv is not None else None,
                        seed, stream, dist,
                        cm.ctypes.data if cm is not None else None, pad_bits)
    if rc != 0:
        raise RuntimeError("synth_fill failed")
    return out


def pick_channels(groups, n, n_pick, seed, stream=STREAM_PICK):
    lib = _load()
    out = np.empty((groups, n_pick), dtype=np.int32)
    if lib.synth_pick_channels(out.ctypes.data, groups, n, n_pick, seed, stream) != 0:
        raise RuntimeError("synth_pick_channels failed")
    return out


def uniform_ints(n, lo, hi, seed, stream=STREAM_LENS):
    lib = _load()
    out = np.empty((n,), dtype=np.int32)
    if lib.synth_uniform_ints(out.ctypes.data, n, lo, hi, seed, stream) != 0:
        raise RuntimeError("synth_uniform_ints failed")
    return out


def num_threads() -> int:
    return int(_load().synth_num_threads())


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass
class Workload:
    """One seeded synthetic attention workload.

    kind      'prefill' (Sq query tokens per sequence attend to Lk keys) or
              'decode' (Sq = nq query tokens per sequence at the end of a KV cache)
    q_dist    DIST_NORMAL or DIST_STUDENT_T3 (likewise k_dist, v_dist)
    k_outliers / q_outliers: number of channels per kv-head scaled by `outlier_mult`
    len_range (lo, hi): per-sequence KV lengths drawn uniformly, else all Lk
    """
    name: str
    kind: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Lk: int
    d: int = 128
    causal: bool = True
    seed: int = 0
    q_dist: int = DIST_NORMAL
    k_dist: int = DIST_NORMAL
    v_dist: int = DIST_NORMAL
    k_outliers: int = 0
    q_outliers: bool = False
    outlier_mult: float = 1.0
    len_range: Optional[tuple] = None
    description: str = ""

    @property
    def G(self):
        return self.Hq // self.Hkv

    def seqlens(self) -> np.ndarray:
        if self.len_range is None:
            return np.full((self.B,), self.Lk, dtype=np.int32)
        lo, hi = self.len_range
        return uniform_ints(self.B, lo, hi, self.seed)

    def outlier_channels(self) -> Optional[np.ndarray]:
        if self.k_outliers <= 0:
            return None
        return pick_channels(self.Hkv, self.d, self.k_outliers, self.seed)

    def generate(self, pad_bits: int = 0):
        """Return dict(q, k, v) of bf16 bit arrays and seqlens (int32[B]).

        q: [B, Sq, Hq, d]; k, v: [B, Lk, Hkv, d]. Tokens of k and v at or past
        seqlens[b] hold `pad_bits`.
        """
        lens = self.seqlens()
        ch = self.outlier_channels()
        k_mult = q_mult = None
        if ch is not None:
            k_mult = np.ones((self.Hkv, self.d), dtype=np.float32)
            for h in range(self.Hkv):
                k_mult[h, ch[h]] = self.outlier_mult
            if self.q_outliers:
                q_mult = np.ones((self.Hq, self.d), dtype=np.float32)
                for hq in range(self.Hq):
                    q_mult[hq, ch[hq // self.G]] = self.outlier_mult
        q = fill(self.B, self.Sq, self.Hq, self.d, self.seed, STREAM_Q, self.q_dist, q_mult)
        k = fill(self.B, self.Lk, self.Hkv, self.d, self.seed, STREAM_K, self.k_dist, k_mult, lens, pad_bits)
        v = fill(self.B, self.Lk, self.Hkv, self.d, self.seed, STREAM_V, self.v_dist, None, lens, pad_bits)
        return dict(q=q, k=k, v=v, seqlens=lens, outlier_channels=ch)


# The five benchmark workloads (bf16 inputs, d = 128).
WORKLOADS = {
    "prefill_b1_h2_s256": Workload(
        "prefill_b1_h2_s256", "prefill", B=1, Hq=2, Hkv=2, Sq=256, Lk=256, causal=True, seed=0,
        description="causal prefill, B=1, Hq=Hkv=2, S=256, N(0,1)"),
    "decode_gqa_b32_hq32_hkv8_l8192": Workload(
        "decode_gqa_b32_hq32_hkv8_l8192", "decode", B=32, Hq=32, Hkv=8, Sq=1, Lk=8192, causal=True,
        seed=1, k_outliers=4, q_outliers=True, outlier_mult=16.0,
        description="GQA decode, 1 query token, KV 8192, 4 outlier channels x16 in Q and K"),
    "prefill_gqa_b4_hq32_hkv8_s8192": Workload(
        "prefill_gqa_b4_hq32_hkv8_s8192", "prefill", B=4, Hq=32, Hkv=8, Sq=8192, Lk=8192, causal=True,
        seed=2, k_outliers=2, q_outliers=False, outlier_mult=20.0,
        description="causal GQA prefill, S=8192, 2 outlier channels x20 in K, quantize timed"),
    "decode_long_b8_hq64_hkv8_l64k_128k": Workload(
        "decode_long_b8_hq64_hkv8_l64k_128k", "decode", B=8, Hq=64, Hkv=8, Sq=1, Lk=131072, causal=True,
        seed=3, q_dist=DIST_STUDENT_T3, k_dist=DIST_STUDENT_T3, len_range=(65536, 131072),
        description="long-context decode, KV lengths U[65536,131072], Student-t(3) Q/K"),
    "verify_b64_nq8_hq64_hkv8_l16384": Workload(
        "verify_b64_nq8_hq64_hkv8_l16384", "decode", B=64, Hq=64, Hkv=8, Sq=8, Lk=16384, causal=True,
        seed=4, k_outliers=4, q_outliers=False, outlier_mult=16.0,
        description="speculative verify, 8 query tokens causal within block, KV 16384, 4 outlier channels x16 in K"),
}

WORKLOAD_ORDER = list(WORKLOADS)
