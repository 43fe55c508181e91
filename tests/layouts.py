"""Rearrange the library's packed layouts into the oracle's logical layouts.

Test code only. Each function is plain indexing, following the layouts that
include/qk4v8.h documents.
"""
import numpy as np


def qk_scales_logical(scales: np.ndarray, T: int) -> np.ndarray:
    """[B, H, cap/128, 512] scale atoms -> [B, H, T, 4] (token t, channel group g)."""
    B, H, nblk, _ = scales.shape
    t = np.arange(T)[:, None]
    g = np.arange(4)[None, :]
    idx = (t // 128) * 512 + (t % 32) * 16 + ((t % 128) // 32) * 4 + g
    return scales.reshape(B, H, nblk * 512)[:, :, idx]


def v_scales_logical(scales: np.ndarray, T: int) -> np.ndarray:
    """[B, H, cap/128, 512] scale atoms -> [B, H, 128, ceil(T/32)] (channel c, token group G)."""
    B, H, nblk, _ = scales.shape
    c = np.arange(128)[:, None]
    G = np.arange((T + 31) // 32)[None, :]
    idx = (G // 4) * 512 + (c % 32) * 16 + (c // 32) * 4 + (G % 4)
    return scales.reshape(B, H, nblk * 512)[:, :, idx]


def v_codes_logical(codes: np.ndarray) -> np.ndarray:
    """Blocked V codes [B, H, cap/128, 128, w] (w = 128 bytes per channel row of a
    block for MXFP8, 64 for MXFP4) -> channel rows [B, H, 128, cap/128 * w]."""
    B, H, nb, C, w = codes.shape
    return np.transpose(codes, (0, 1, 3, 2, 4)).reshape(B, H, C, nb * w)


def fill_v_bytes(codes, b, start, value, stop=None):
    """Sets the token-axis bytes [start, stop) of batch entry b, every head and
    channel, of blocked V codes [B, H, cap/128, 128, w] (torch or numpy; bytes are
    tokens for MXFP8, token pairs for MXFP4). stop defaults to the capacity."""
    nb, w = codes.shape[2], codes.shape[4]
    stop = nb * w if stop is None else stop
    for blk in range(start // w, (stop + w - 1) // w):
        lo, hi = max(start - blk * w, 0), min(stop - blk * w, w)
        if lo < hi:
            codes[b, :, blk, :, lo:hi] = value


def unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    """[..., 64] bytes -> [..., 128] codes, element 2i from the low nibble of byte i."""
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def gather_pages(codes, scales, block_table, n_blocks):
    """Paged pools -> contiguous packed tensors of n_blocks 128-token blocks.

    codes [P, H, R, X] and scales [P, H, 512] (numpy), block_table [B, max_pages].
    K pools (R = 128 tokens, X = 64 bytes) give codes [B, H, n_blocks * 128, 64];
    V pools (R = 128 channels, X = 128 tokens) give codes [B, H, 128, n_blocks * 128].
    Scales come back as [B, H, n_blocks, 512] atoms. Plain indexing."""
    idx = np.asarray(block_table)[:, :n_blocks]
    c = codes[idx]                                   # [B, n, H, R, X]
    s = scales[idx]                                  # [B, n, H, 512]
    B, n, H, R, X = c.shape
    if X == 64:      # K: token rows
        c = np.transpose(c, (0, 2, 1, 3, 4)).reshape(B, H, n * R, X)
    else:            # V: channel rows, tokens contiguous
        c = np.transpose(c, (0, 2, 3, 1, 4)).reshape(B, H, R, n * X)
    return c, np.transpose(s, (0, 2, 1, 3))
