// Paged KV cache append with online scale update.
//
// MpFA QK4V8 article, section 3.2: the block scales are computed online, from
// the data of the block itself, with no calibration; section 6.1: the QK4V8
// attention runs over a quantized KV cache. Decode appends tokens to that
// cache one step at a time (1 token, or the 8 tokens of a verified draft
// block), into pages of 128 tokens taken from a pool (paged attention).
//
// K is quantized per token (one MXFP4 scale per 32 channels), so a new token's
// K row is encoded on its own and written into its page. V is quantized per
// channel over groups of 32 tokens along the sequence: a token that lands in a
// group that already holds tokens changes that group's amax, so the group's
// scale is recomputed and every code of the group re-encoded. To do that
// exactly (the result is identical to quantizing the whole sequence at once),
// the bf16 values of the open group, the last, partly filled group of each
// (sequence, KV head), are kept in a small staging buffer ("tail", 32 tokens x
// 128 channels of bf16) that the append reads and refreshes.
//
// Page layout (one page = 128 tokens of one KV head, as the contiguous layout
// with capacity 128):
//   K codes  [pages][Hkv][128][64],  K scales [pages][Hkv][512]
//   V codes  [pages][Hkv][128][128] (channel rows, token-contiguous),
//   V scales [pages][Hkv][512]
// Token t of sequence b lives in page block_table[b][t / 128] at row t % 128.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/qk4v8.h"
#include "mx_encode.cuh"
#include "ptx.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

namespace {

__device__ __forceinline__ void flag_bad_page(int32_t *status) {
    if (status) atomicCAS(status, 0, QK4V8_ERR_INVALID_ARG);
}

// Page of token position pos of sequence b, or -1 if the block table has no
// valid page there.
__device__ __forceinline__ int page_of(const int32_t *__restrict__ block_table, int max_pages, int num_pages, int b,
                                       int pos) {
    const int slot = pos >> 7;
    if (pos < 0 || slot >= max_pages) return -1;
    const int page = block_table[static_cast<int64_t>(b) * max_pages + slot];
    return (page >= 0 && page < num_pages) ? page : -1;
}

}  // namespace

// One kernel does the whole append. CTA (b, h, chunk), 128 threads:
//  - K: the chunk's share of the n_new rows of head h, 16 lanes per row (two
//    rows per warp step), with the quantization kernels' encoder (identical
//    bytes), optionally after the Hadamard rotation of the row;
//  - V: thread c = channel c; the chunk's share of the 32-token groups the new
//    tokens touch. A group's tokens come from the staging buffer (those before
//    the append, only in the first touched group) and from the new rows; the
//    channel's amax over them fixes the E8M0 scale, all of the group's codes
//    are (re)written, and codes past the new length are zero;
//  - chunk 0 then refreshes the staging buffer with the open group after the
//    append. It is also the only reader of the old staging (the first touched
//    group is its own), and thread c reads and writes only column c, so the
//    refresh needs no barrier;
//  - with a separate seqlens_out, CTA (b, 0, 0) writes the new length (no CTA
//    reads seqlens_out). When the two are the same array, a second launch
//    advances the lengths after every reader.
template <bool kRotate>
__global__ void __launch_bounds__(128) kv_append_kernel(const __nv_bfloat16 *__restrict__ k,
                                                        const __nv_bfloat16 *__restrict__ v, int n_new, int H,
                                                        int64_t sb, int64_t st, int64_t sh,
                                                        const int32_t *__restrict__ seqlens,
                                                        const int32_t *__restrict__ block_table, int max_pages,
                                                        int num_pages, uint8_t *__restrict__ k_codes,
                                                        uint8_t *__restrict__ k_scales, uint8_t *__restrict__ v_codes,
                                                        uint8_t *__restrict__ v_scales, __nv_bfloat16 *__restrict__ tail,
                                                        int chunks, int32_t *seqlens_out, int32_t *status) {
    const int ci = static_cast<int>(blockIdx.x % chunks);
    const int h = static_cast<int>((blockIdx.x / chunks) % H);
    const int b = static_cast<int>(blockIdx.x / (static_cast<int64_t>(chunks) * H));
    const int L0 = seqlens[b];
    const int L1 = L0 + n_new;
    const int c = threadIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // ---- K rows [r_begin, r_end) of this chunk
    const int rows_per_chunk = (n_new + chunks - 1) / chunks;
    const int r_begin = ci * rows_per_chunk;
    const int r_end = r_begin + rows_per_chunk < n_new ? r_begin + rows_per_chunk : n_new;
    const int sub = lane & 15;
    // The loop bound is per warp, so all 32 lanes reach the encoder's shuffles.
    for (int r0 = r_begin + 2 * warp; r0 < r_end; r0 += 8) {
        const int t = r0 + (lane >> 4);
        const bool in = t < r_end;
        const int pos = L0 + t;
        int page = -1;
        if (in) {
            page = page_of(block_table, max_pages, num_pages, b, pos);
            if (page < 0 && sub == 0) flag_bad_page(status);
        }
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (page >= 0) raw = *reinterpret_cast<const uint4 *>(k + b * sb + t * st + h * sh + sub * 8);
        int X;
        uint32_t packed;
        if (kRotate) {
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            float x[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[2 * i] = __uint_as_float(w[i] << 16);
                x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
            hadamard128_rows(x, sub);
            packed = mxfp4_encode8_f32(x, true, X);
        } else {
            packed = mxfp4_encode8(raw, true, X);
        }
        if (page >= 0) {
            const int64_t row = static_cast<int64_t>(page) * H + h;
            const int rr = pos & 127;
            reinterpret_cast<uint32_t *>(k_codes + (row * 128 + rr) * 64)[sub] = packed;
            if ((sub & 3) == 0)
                k_scales[row * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (sub >> 2)] = static_cast<uint8_t>(X + 127);
        }
    }

    // ---- V groups L0 / 32 + ci, + chunks, ... touched by the new tokens
    uint16_t *tail_bh = reinterpret_cast<uint16_t *>(tail) + ((static_cast<int64_t>(b) * H + h) * 32) * 128;
    const uint16_t *vin = reinterpret_cast<const uint16_t *>(v) + b * sb + h * sh + c;
    for (int G = L0 / 32 + ci; G * 32 < L1; G += chunks) {
        const int t0 = G * 32;
        const int page = page_of(block_table, max_pages, num_pages, b, t0);
        if (page < 0) {
            if (c == 0) flag_bad_page(status);
            continue;
        }
        uint16_t x[32];
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int t = t0 + j;
            uint16_t bits = 0;
            if (t < L0)
                bits = tail_bh[j * 128 + c];  // staged before this append
            else if (t < L1)
                bits = vin[(t - L0) * st];
            x[j] = bits;
            amax = fmaxf(amax, fabsf(__uint_as_float(static_cast<uint32_t>(bits) << 16)));
        }
        const int X = shared_exponent(amax, 8);
        const float f = pow2_neg(X);
        // x / 2^X is exact; the conversion keeps the sign bit, also of a value
        // that rounds to zero. Tokens past L1 encode as zero.
        uint32_t words[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const uint32_t lo = cvt_e4m3x2(__uint_as_float(static_cast<uint32_t>(x[4 * q]) << 16) * f,
                                           __uint_as_float(static_cast<uint32_t>(x[4 * q + 1]) << 16) * f);
            const uint32_t hi = cvt_e4m3x2(__uint_as_float(static_cast<uint32_t>(x[4 * q + 2]) << 16) * f,
                                           __uint_as_float(static_cast<uint32_t>(x[4 * q + 3]) << 16) * f);
            words[q] = lo | (hi << 16);
        }
        const int64_t row = static_cast<int64_t>(page) * H + h;
        uint4 *dst = reinterpret_cast<uint4 *>(v_codes + (row * 128 + c) * 128 + (t0 & 127));
        dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
        dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
        v_scales[row * 512 + (c & 31) * 16 + (c >> 5) * 4 + ((t0 >> 5) & 3)] = static_cast<uint8_t>(X + 127);
    }

    // ---- the open group after the append, staged in slots t % 32 (its tokens
    // from before the append are in place already)
    if (ci == 0 && (L1 & 31) != 0) {
        const int t0 = L1 & ~31;
        for (int t = t0 > L0 ? t0 : L0; t < L1; ++t) tail_bh[(t - t0) * 128 + c] = vin[(t - L0) * st];
    }
    if (seqlens_out && ci == 0 && h == 0 && c == 0) seqlens_out[b] = L1;
}

// seqlens[b] += n_new in place, after every reader of seqlens ran.
__global__ void kv_advance_lengths_kernel(int32_t *seqlens, int B, int n_new) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) seqlens[b] += n_new;
}

cudaError_t launch_kv_append(const void *k, const void *v, int B, int n_new, int H, int64_t sb, int64_t st,
                             int64_t sh, const int32_t *seqlens, const int32_t *block_table, int max_pages,
                             int num_pages, uint8_t *k_codes, uint8_t *k_scales, uint8_t *v_codes,
                             uint8_t *v_scales, void *tail, bool rotate_k, int32_t *seqlens_out, int32_t *status,
                             cudaStream_t stream) {
    // Chunks per (sequence, head): at most 8 touched V groups and 256 K rows
    // per CTA (one chunk for a decode step of up to 32 tokens).
    const int groups = (n_new + 31) / 32 + 1;  // the open group and those the new tokens fill
    int chunks = (groups + 7) / 8;
    const int chunks_k = (n_new + 255) / 256;
    if (chunks_k > chunks) chunks = chunks_k;
    const int64_t grid = static_cast<int64_t>(B) * H * chunks;
    if (grid >= (int64_t{1} << 31)) return cudaErrorInvalidValue;
    const bool in_place = seqlens_out && seqlens_out == seqlens;
    int32_t *direct_out = in_place ? nullptr : seqlens_out;
    const __nv_bfloat16 *kk = static_cast<const __nv_bfloat16 *>(k);
    const __nv_bfloat16 *vv = static_cast<const __nv_bfloat16 *>(v);
    __nv_bfloat16 *tl = static_cast<__nv_bfloat16 *>(tail);
    if (rotate_k)
        kv_append_kernel<true><<<static_cast<unsigned>(grid), 128, 0, stream>>>(
            kk, vv, n_new, H, sb, st, sh, seqlens, block_table, max_pages, num_pages, k_codes, k_scales, v_codes,
            v_scales, tl, chunks, direct_out, status);
    else
        kv_append_kernel<false><<<static_cast<unsigned>(grid), 128, 0, stream>>>(
            kk, vv, n_new, H, sb, st, sh, seqlens, block_table, max_pages, num_pages, k_codes, k_scales, v_codes,
            v_scales, tl, chunks, direct_out, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !in_place) return e;
    kv_advance_lengths_kernel<<<(B + 255) / 256, 256, 0, stream>>>(seqlens_out, B, n_new);
    return cudaGetLastError();
}

}  // namespace qk4v8
