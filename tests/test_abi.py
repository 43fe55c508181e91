"""The C ABI without a GPU: the library loads, every declared symbol is exported
and bound, the size helpers agree with the documented layouts, and bad
arguments are rejected before any device work."""
import ctypes
import os
import re
import subprocess

import pytest

import bit_quantized_attention_qk4v8_b200 as qk
from bit_quantized_attention_qk4v8_b200 import _lib
from bit_quantized_attention_qk4v8_b200 import build as qkbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in ("qk4v8.h", "qk4v8_test.h"):
        text = open(os.path.join(ROOT, "include", h)).read()
        names += re.findall(r"QK4V8_API\s+[\w\s\*]+?\b(qk4v8_\w+)\s*\(", text)
    return names


@pytest.fixture(scope="module")
def lib():
    qkbuild.build()
    return _lib.lib()


def test_library_is_not_stale(lib):
    """The built libqk4v8.so is newer than every source it is built from."""
    assert not qkbuild._stale()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    nm = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\sT\s+(\w+)", nm.stdout))
    for n in names:
        assert n in exported, n
        assert n in _lib.SIGNATURES, f"{n} has no Python binding"
        getattr(lib, n)
    # nothing exported that the headers do not declare
    assert {e for e in exported if e.startswith("qk4v8_")} == set(names)


def test_size_helpers(lib):
    assert lib.qk4v8_mxfp4_codes_bytes(2, 3, 256) == 2 * 3 * 256 * 64
    assert lib.qk4v8_mxfp8_codes_bytes(2, 3, 256) == 2 * 3 * 128 * 256
    assert lib.qk4v8_scales_bytes(2, 3, 256) == 2 * 3 * 2 * 512
    assert lib.qk4v8_decode_workspace_bytes(4, 8, 2, 3) == 4 * 8 * 2 * 3 * 129 * 4 + 4 * 8 * 4
    assert lib.qk4v8_decode_workspace_bytes(0, 8, 2, 3) == 0
    # KV bytes per token per kv-head: 64 (E2M1 codes) + 128 (E4M3) + 4 + 4 (scales) = 200
    cap = 8192
    per_tok = (lib.qk4v8_mxfp4_codes_bytes(1, 1, cap) + lib.qk4v8_mxfp8_codes_bytes(1, 1, cap)
               + 2 * lib.qk4v8_scales_bytes(1, 1, cap)) / cap
    assert per_tok == 200.0


def test_default_splits(lib):
    """148 SMs without a device. For 33..64 rows per KV head (the persistent GQA
    decode kernel), with at most half as many sequences as CTAs and at least two
    key tiles per CTA: enough splits for its balanced schedule with sequences of
    half the maximum length, ceil(tiles / half) + 1 with half = units * tiles /
    slots / 2. Worked by hand: B=8, Hkv=8, 64 rows (one CTA per SM, 148 slots),
    1024 tiles: half = 65536 / 148 / 2 = 221, so 5 + 1 = 6. Otherwise the wave
    cost model, waves * (tiles per split + 3): B=32, Hkv=8, 4 rows (two CTAs per
    SM, 296 slots), 64 tiles: s=1 costs 1 * 67, s=2 costs 2 * 35. B=8, Hkv=8,
    8 rows, 1024 tiles: s=9 is 576 CTAs in 2 waves of 114 + 3 = 234, below s=4
    (259) and s=18 (240). B=64, Hkv=8, 64 rows, 128 tiles: s=2 is 7 waves of
    67 = 469, below s=1 (4 * 131) and s=4 (14 * 35)."""
    f = lib.qk4v8_decode_default_splits
    assert f(32, 32, 8, 1, 8192) == 1
    assert f(8, 64, 8, 1, 131072) == 9
    assert f(8, 64, 8, 8, 131072) == 6
    assert f(64, 64, 8, 8, 16384) == 2
    assert f(1, 1, 1, 1, 100) == 1
    assert f(2, 8, 2, 1, 1000) == 8          # wave model; never more splits than tiles
    for bad in ((0, 8, 8, 1, 100), (1, 30, 8, 1, 100), (1, 8, 8, 0, 100)):
        assert f(*bad) == 1


def test_plan_splits(lib):
    """The length-aware plan (148 SMs without a device; two CTAs per SM up to 16
    rows: 296 slots). Worked by hand for two sequences of 10 and 1 tiles, 4 rows,
    one KV head: every CTA runs at the 1.5x single-CTA rate (2..11 CTAs on 296
    slots). s=1: the 1-tile CTA ends at 1/1.5, the 10-tile one at 10/1.5 = 6.67,
    plus the launch (17): 23.67. s=10 (1 tile per split): 11 CTAs all end at
    0.67, plus launch and merge (17 + 4): 21.67, the least (s=5: 1.33 + 21).
    For 33..64 rows it is the default plan; invalid sizes give 1."""
    import ctypes
    import numpy as np

    def plan(B, Hq, Hkv, nq, lens, window=0):
        a = np.ascontiguousarray(lens, dtype=np.int32)
        return lib.qk4v8_decode_plan_splits(B, Hq, Hkv, nq, a.ctypes.data_as(ctypes.c_void_p), window)

    assert plan(2, 4, 1, 1, [1280, 128]) == 10
    # Window 128: the tiles are counted from the window's first key, 2 and 1 here:
    # s=1 ends at 2/1.5 + 17 = 18.3, s=2 (three 1-tile CTAs) at 1/1.5 + 17 + 4 = 21.7.
    assert plan(2, 4, 1, 1, [1280, 128], window=128) == 1
    assert plan(32, 32, 8, 1, [8192] * 32) == 1
    assert plan(64, 64, 8, 8, [16384] * 64) == lib.qk4v8_decode_default_splits(64, 64, 8, 8, 16384)
    assert plan(0, 4, 1, 1, [1]) == 1
    assert lib.qk4v8_decode_plan_splits(2, 4, 1, 1, None, 0) == 1


FAKE = 0x10000  # never dereferenced: validation rejects these calls first


def test_quantize_rejects_bad_args(lib):
    args = dict(x=FAKE, B=1, S=10, H=2, d=128, sb=2560, ss=256, sh=128, sl=None, cap=128, c=FAKE, s=FAKE)

    def call(**kw):
        a = dict(args, **kw)
        return lib.qk4v8_quantize_qk(a["x"], a["B"], a["S"], a["H"], a["d"], a["sb"], a["ss"], a["sh"], a["sl"],
                                     a["cap"], a["c"], a["s"], None)

    assert call(d=64) == 1
    assert call(x=None) == 1
    assert call(cap=100) == 1
    assert call(cap=0) == 1
    assert call(S=129, cap=128) == 1
    assert call(x=FAKE + 4) == 1
    assert call(ss=250) == 1
    assert b"head_dim" in lib.qk4v8_last_error() or True


def test_decode_rejects_bad_args(lib):
    def call(nq=1, Hq=32, Hkv=8, seqlens=FAKE, ws=FAKE, wsb=10**9, max_len=8192, kv_cap=8192, splits=0):
        return lib.qk4v8_attention_decode(FAKE, FAKE, 2, Hq, nq, 128, FAKE, FAKE, FAKE, FAKE, Hkv, kv_cap, seqlens,
                                          max_len, 1, 0.0, splits, ws, wsb, FAKE, None, None, None)

    assert call(nq=9) == 1
    assert call(nq=0) == 1
    assert call(Hq=64, Hkv=1, nq=4) == 1      # 64 * 4 rows > 128
    assert call(Hq=30, Hkv=8) == 1            # Hq % Hkv
    assert call(seqlens=None) == 1
    assert call(wsb=16) == 1                  # workspace too small
    assert call(max_len=9000) == 1            # beyond kv_cap
    assert call(kv_cap=1000, max_len=900) == 1
    assert call(splits=-1) == 1
    assert b"workspace" in lib.qk4v8_last_error() or True


def test_bf16_decode_workspace_bytes(lib):
    f = lib.qk4v8_decode_bf16_workspace_bytes
    part = lib.qk4v8_decode_workspace_bytes
    assert f(32, 32, 8, 1, 1) == 0                      # 4 rows, one split: written directly, no scratch
    assert f(32, 32, 8, 1, 3) == part(32, 32, 1, 3)      # partials for the merge
    assert f(2, 32, 8, 8, 1) == 0                        # 32 rows: quantized inside the swap-AB kernel
    packed_64 = 2 * 64 * 128 * 64 + 2 * 64 * 512          # 33..64 rows: MXFP4 Q, capacity 128, in front
    assert f(2, 64, 8, 8, 1) == packed_64                # one split: the GQA decode kernel writes out directly
    assert f(2, 64, 8, 8, 2) == packed_64 + part(2, 64, 8, 2)
    packed_q = 2 * 128 * 128 * 64 + 2 * 128 * 512         # 128 rows: MXFP4 Q, capacity 128, in front
    assert f(2, 128, 8, 8, 2) == packed_q + part(2, 128, 8, 2)
    assert f(0, 8, 8, 1, 1) == 0 and f(1, 30, 8, 1, 1) == 0


def test_bf16_decode_rejects_bad_args(lib):
    def call(q=FAKE, nq=1, Hq=32, Hkv=8, sb=32 * 128, st=32 * 128, sh=128, splits=1, ws=None, wsb=0, out=FAKE):
        return lib.qk4v8_attention_decode_bf16(q, 2, Hq, nq, sb, st, sh, FAKE, FAKE, FAKE, FAKE, Hkv, 8192, FAKE,
                                               8192, 1, 0.0, splits, ws, wsb, out, None, None, None)

    assert call(q=None) == 1
    assert call(nq=9) == 1
    assert call(Hq=64, Hkv=1, nq=4) == 1      # 256 rows
    assert call(out=FAKE + 2) == 1
    assert call(splits=3) == 1                # partials need a workspace
    assert call(q=FAKE + 2) == 1              # bf16 rows must be 16-byte aligned
    assert call(sh=100) == 1                  # strides in whole 16-byte units


def test_prefill_rejects_bad_args(lib):
    def call(Sq=256, q_cap=256, Sk=256, kv_cap=256, Hq=4, Hkv=2, out=FAKE):
        return lib.qk4v8_attention_prefill(FAKE, FAKE, 1, Hq, Sq, q_cap, FAKE, FAKE, FAKE, FAKE, Hkv, Sk, kv_cap,
                                           None, 1, 0.0, out, None, None, None)

    assert call(q_cap=200) == 1
    assert call(Sq=300) == 1
    assert call(Sk=300) == 1
    assert call(Hq=3) == 1
    assert call(out=None) == 1
    assert call(out=FAKE + 2) == 1


def test_status_strings(lib):
    for st in range(5):
        assert lib.qk4v8_status_string(st)
    assert lib.qk4v8_status_string(4) == b"device wait timed out"


def test_binding_raises_without_cuda_tensors():
    import torch
    with pytest.raises(ValueError):
        qk.quantize_qk(torch.zeros((1, 4, 1, 128), dtype=torch.bfloat16))
