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

// K rows: 16 lanes per (sequence, new token, head) row, two rows per warp step,
// the encoder of the quantization kernels (identical bytes), optionally after
// the Hadamard rotation of the row.
template <bool kRotate>
__global__ void __launch_bounds__(256) kv_append_k_kernel(const __nv_bfloat16 *__restrict__ k, int B, int n_new,
                                                          int H, int64_t sb, int64_t st, int64_t sh,
                                                          const int32_t *__restrict__ seqlens,
                                                          const int32_t *__restrict__ block_table, int max_pages,
                                                          int num_pages, uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ scales, int32_t *status) {
    const int sub = threadIdx.x & 15;
    const int64_t rows = static_cast<int64_t>(B) * n_new * H;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t base = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 2;
         base < rows; base += 2 * warps) {
        const int64_t r = base + ((threadIdx.x >> 4) & 1);
        const bool in = r < rows;
        int b = 0, t = 0, h = 0, page = -1, pos = 0;
        if (in) {
            h = static_cast<int>(r % H);
            t = static_cast<int>((r / H) % n_new);
            b = static_cast<int>(r / (static_cast<int64_t>(H) * n_new));
            pos = seqlens[b] + t;
            page = page_of(block_table, max_pages, num_pages, b, pos);
            if (page < 0 && sub == 0) flag_bad_page(status);
        }
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (page >= 0) raw = *reinterpret_cast<const uint4 *>(k + b * sb + t * st + h * sh + sub * 8);
        int X;
        uint32_t packed;
        if (kRotate) {
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __uint_as_float(w[i] << 16);
                v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
            hadamard128_rows(v, sub);
            packed = mxfp4_encode8_f32(v, true, X);
        } else {
            packed = mxfp4_encode8(raw, true, X);
        }
        if (page >= 0) {
            const int64_t row = static_cast<int64_t>(page) * H + h;
            const int rr = pos & 127;
            reinterpret_cast<uint32_t *>(codes + (row * 128 + rr) * 64)[sub] = packed;
            if ((sub & 3) == 0)
                scales[row * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (sub >> 2)] = static_cast<uint8_t>(X + 127);
        }
    }
}

// V: one CTA of 128 threads (one per channel) per (sequence, head, touched
// 32-token group). The group's tokens come from the staging buffer (those
// before the append) and from the new rows; the channel's amax over them
// fixes the E8M0 scale, all of the group's codes are (re)written, and codes
// past the new length are zero. The staging buffer is refreshed afterwards by
// kv_tail_update_kernel (a separate launch: the CTA of the first group reads
// slots that the last group's new tokens take).
__global__ void __launch_bounds__(128) kv_append_v_kernel(const __nv_bfloat16 *__restrict__ v, int B, int n_new,
                                                          int H, int64_t sb, int64_t st, int64_t sh,
                                                          const int32_t *__restrict__ seqlens,
                                                          const int32_t *__restrict__ block_table, int max_pages,
                                                          int num_pages, uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ scales,
                                                          const __nv_bfloat16 *__restrict__ tail, int groups_per_seq,
                                                          int32_t *status) {
    const int c = threadIdx.x;
    const int gi = static_cast<int>(blockIdx.x % groups_per_seq);
    const int h = static_cast<int>((blockIdx.x / groups_per_seq) % H);
    const int b = static_cast<int>(blockIdx.x / (static_cast<int64_t>(groups_per_seq) * H));
    const int L0 = seqlens[b];
    const int L1 = L0 + n_new;
    const int G = L0 / 32 + gi;       // the group this CTA writes
    if (G * 32 >= L1) return;         // fewer groups touched than the grid allows for
    const int t0 = G * 32;
    const int page = page_of(block_table, max_pages, num_pages, b, t0);
    if (page < 0) {
        if (c == 0) flag_bad_page(status);
        return;
    }
    const __nv_bfloat16 *tail_bh = tail + ((static_cast<int64_t>(b) * H + h) * 32) * 128;
    const uint16_t *vin = reinterpret_cast<const uint16_t *>(v) + b * sb + h * sh + c;
    uint16_t x[32];
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int t = t0 + j;
        uint16_t bits = 0;
        if (t < L0)
            bits = reinterpret_cast<const uint16_t *>(tail_bh)[j * 128 + c];   // staged before this append
        else if (t < L1)
            bits = vin[(t - L0) * st];
        x[j] = bits;
        amax = fmaxf(amax, fabsf(__uint_as_float(static_cast<uint32_t>(bits) << 16)));
    }
    const int X = shared_exponent(amax, 8);
    const float f = pow2_neg(X);
    uint32_t words[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
            const uint32_t b0 = x[4 * q + e], b1 = x[4 * q + e + 1];
            uint32_t pair = cvt_e4m3x2(fabsf(__uint_as_float(b0 << 16)) * f, fabsf(__uint_as_float(b1 << 16)) * f);
            pair |= ((b0 >> 15) & 1u) << 7;
            pair |= ((b1 >> 15) & 1u) << 15;
            word |= pair << (8 * e);
        }
        words[q] = word;
    }
    // Tokens past L1 encode as zero (their inputs were zero, and a zero keeps
    // code 0 whatever the scale).
    const int64_t row = static_cast<int64_t>(page) * H + h;
    uint4 *dst = reinterpret_cast<uint4 *>(codes + (row * 128 + c) * 128 + (t0 & 127));
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    scales[row * 512 + (c & 31) * 16 + (c >> 5) * 4 + ((t0 >> 5) & 3)] = static_cast<uint8_t>(X + 127);
}

// The open group after the append (tokens 32 * (L1 / 32) .. L1 - 1), staged in
// slots t % 32: its tokens from before the append are in place already; the
// new ones are copied in. One CTA of 128 threads (channels) per (sequence,
// head).
__global__ void __launch_bounds__(128) kv_tail_update_kernel(const __nv_bfloat16 *__restrict__ v, int n_new, int H,
                                                             int64_t sb, int64_t st, int64_t sh,
                                                             const int32_t *__restrict__ seqlens,
                                                             __nv_bfloat16 *__restrict__ tail) {
    const int c = threadIdx.x;
    const int h = static_cast<int>(blockIdx.x % H);
    const int b = static_cast<int>(blockIdx.x / H);
    const int L0 = seqlens[b];
    const int L1 = L0 + n_new;
    if ((L1 & 31) == 0) return;  // no open group
    const int t0 = L1 & ~31;
    uint16_t *tail_bh = reinterpret_cast<uint16_t *>(tail) + ((static_cast<int64_t>(b) * H + h) * 32) * 128;
    const uint16_t *vin = reinterpret_cast<const uint16_t *>(v) + b * sb + h * sh + c;
    for (int t = t0 > L0 ? t0 : L0; t < L1; ++t) tail_bh[(t - t0) * 128 + c] = vin[(t - L0) * st];
}

// seqlens_out[b] = seqlens[b] + n_new, after every reader of seqlens ran (the
// two may be the same array).
__global__ void kv_advance_lengths_kernel(const int32_t *seqlens, int B, int n_new, int32_t *seqlens_out) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) seqlens_out[b] = seqlens[b] + n_new;
}

cudaError_t launch_kv_append(const void *k, const void *v, int B, int n_new, int H, int64_t sb, int64_t st,
                             int64_t sh, const int32_t *seqlens, const int32_t *block_table, int max_pages,
                             int num_pages, uint8_t *k_codes, uint8_t *k_scales, uint8_t *v_codes,
                             uint8_t *v_scales, void *tail, bool rotate_k, int32_t *seqlens_out, int32_t *status,
                             cudaStream_t stream) {
    const int64_t rows = static_cast<int64_t>(B) * n_new * H;
    int64_t grid_k = (rows + 15) / 16;  // 16 rows per CTA (8 warps, two rows each)
    if (grid_k > 148 * 8) grid_k = 148 * 8;
    if (grid_k < 1) grid_k = 1;
    const __nv_bfloat16 *kk = static_cast<const __nv_bfloat16 *>(k);
    if (rotate_k)
        kv_append_k_kernel<true><<<static_cast<unsigned>(grid_k), 256, 0, stream>>>(
            kk, B, n_new, H, sb, st, sh, seqlens, block_table, max_pages, num_pages, k_codes, k_scales, status);
    else
        kv_append_k_kernel<false><<<static_cast<unsigned>(grid_k), 256, 0, stream>>>(
            kk, B, n_new, H, sb, st, sh, seqlens, block_table, max_pages, num_pages, k_codes, k_scales, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // Groups one append can touch: the open one and those the new tokens fill.
    const int groups = (n_new + 31) / 32 + 1;
    const int64_t grid_v = static_cast<int64_t>(B) * H * groups;
    kv_append_v_kernel<<<static_cast<unsigned>(grid_v), 128, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(v), B, n_new, H, sb, st, sh, seqlens, block_table, max_pages, num_pages,
        v_codes, v_scales, static_cast<const __nv_bfloat16 *>(tail), groups, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    kv_tail_update_kernel<<<static_cast<unsigned>(static_cast<int64_t>(B) * H), 128, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(v), n_new, H, sb, st, sh, seqlens, static_cast<__nv_bfloat16 *>(tail));
    e = cudaGetLastError();
    if (e != cudaSuccess || !seqlens_out) return e;
    kv_advance_lengths_kernel<<<(B + 255) / 256, 256, 0, stream>>>(seqlens, B, n_new, seqlens_out);
    return cudaGetLastError();
}

}  // namespace qk4v8
