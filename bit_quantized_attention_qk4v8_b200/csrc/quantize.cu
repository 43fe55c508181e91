// MX quantization kernels: bf16 Q/K -> MXFP4, bf16 V -> MXFP8-E4M3.
//
// MpFA QK4V8 article: Q and K go to 4 bits, V to 8 bits (sections 1.1,
// 2.1-2.2), with each block's scale computed online as the block is read,
// without calibration (sections 1.2, 3.2). MiMo FP4 article, "MXFP4专家量化":
// one block scale per 32 values. The scale rule is OCP MX:
// X = floor(log2 amax) - emax, and each element is rounded to nearest even at
// x / 2^X with saturation. Both kernels are bandwidth bound. They read the
// bf16 tensor once and write the packed codes and scales once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mx_encode.cuh"
#include "ptx.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

// ------------------------------------------------------------------ MXFP4

// 16 lanes per token row (128 channels), 8 channels per lane, 4 lanes per group
// of 32. Rows are visited in input order (b, t, h) so loads are contiguous.
// Tokens 0 .. row_len-1 of each sequence are visited: row_len = cap writes the
// whole capacity (zero codes and scales past the valid length), row_len = S
// only the rows of the input.
__global__ void __launch_bounds__(256) quantize_qk_kernel(const __nv_bfloat16 *__restrict__ x, int B, int S, int H,
                                                          int64_t sb, int64_t ss, int64_t sh,
                                                          const int32_t *__restrict__ seqlens, int cap,
                                                          int row_len, uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ scales) {
    const int sub = threadIdx.x & 15;  // lane within the row
    const int64_t n_rows = static_cast<int64_t>(B) * row_len * H;
    const int64_t row_step = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 4);
    // The loop bound is taken per warp (two rows) so every lane reaches the shuffles.
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 4) + ((threadIdx.x >> 5) << 1);
         base < n_rows; base += row_step) {
        const int64_t row_raw = base + ((threadIdx.x >> 4) & 1);
        const bool in_range = row_raw < n_rows;
        const int64_t row = in_range ? row_raw : base;
        const int h = static_cast<int>(row % H);
        const int64_t bt = row / H;
        const int t = static_cast<int>(bt % row_len);
        const int b = static_cast<int>(bt / row_len);
        int valid_len = S;
        if (seqlens) {
            int L = seqlens[b];
            valid_len = L < valid_len ? L : valid_len;
        }
        const bool valid = in_range && t < valid_len;
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (valid) raw = *reinterpret_cast<const uint4 *>(x + b * sb + t * ss + h * sh + sub * 8);
        int X;
        const uint32_t packed = mxfp4_encode8(raw, valid, X);
        if (!in_range) continue;
        const int64_t head = static_cast<int64_t>(b) * H + h;
        reinterpret_cast<uint32_t *>(codes + (head * cap + t) * 64)[sub] = packed;
        if ((sub & 3) == 0) {
            const int g = sub >> 2;
            uint8_t *blk = scales + (head * (cap / 128) + t / 128) * 512;
            blk[(t & 31) * 16 + ((t & 127) >> 5) * 4 + g] = valid ? static_cast<uint8_t>(X + 127) : 0;
        }
    }
}

// ------------------------------------------------------------------ MXFP8 V

// One CTA per (b, h, 128-token block): stage the bf16 tile in shared memory,
// quantize each channel's four 32-token groups, and write the token-contiguous
// codes plus the block's 512-byte scale atom.
constexpr int kVPitch = 136;  // bf16 elements per staged token row (16-byte padding)
constexpr int kCPitch = 144;  // bytes per staged code row

__global__ void __launch_bounds__(256) quantize_v_kernel(const __nv_bfloat16 *__restrict__ v, int B, int S, int H,
                                                         int64_t sb, int64_t ss, int64_t sh,
                                                         const int32_t *__restrict__ seqlens, int cap,
                                                         uint8_t *__restrict__ codes,
                                                         uint8_t *__restrict__ scales) {
    __shared__ __align__(16) uint16_t tile[128 * kVPitch];  // bf16 staging, later the code tile
    __shared__ __align__(16) uint8_t atom[512];
    uint8_t *ctile = reinterpret_cast<uint8_t *>(tile);     // [128 channels][kCPitch] after the barrier
    const int nblk = cap / 128;
    const int blk = blockIdx.x % nblk;
    const int h = (blockIdx.x / nblk) % H;
    const int b = blockIdx.x / (nblk * H);
    const int t0 = blk * 128;
    int valid_len = S;
    if (seqlens) {
        int L = seqlens[b];
        valid_len = L < valid_len ? L : valid_len;
    }
    // Stage: invalid tokens read as zeros, which leaves them out of every amax
    // and gives them code 0; a group with no valid token gets scale byte 0.
    for (int i = threadIdx.x; i < 128 * 16; i += 256) {
        const int tk = i >> 4, ch = i & 15;
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (t0 + tk < valid_len)
            raw = *reinterpret_cast<const uint4 *>(v + b * sb + static_cast<int64_t>(t0 + tk) * ss + h * sh + ch * 8);
        *reinterpret_cast<uint4 *>(&tile[tk * kVPitch + ch * 8]) = raw;
    }
    __syncthreads();
    const int c = threadIdx.x & 127;
    const int g0 = threadIdx.x >> 7;
    uint32_t words[2][8];
    int Xs[2];
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
        const int g = g0 + 2 * gi;
        float amax = 0.f;
#pragma unroll 8
        for (int j = 0; j < 32; ++j)
            amax = fmaxf(amax, fabsf(__uint_as_float(static_cast<uint32_t>(tile[(g * 32 + j) * kVPitch + c]) << 16)));
        const int X = shared_exponent(amax, 8);
        Xs[gi] = X;
        const float f = pow2_neg(X);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const uint32_t b0 = tile[(g * 32 + 4 * q + e) * kVPitch + c];
                const uint32_t b1 = tile[(g * 32 + 4 * q + e + 1) * kVPitch + c];
                const float y0 = fabsf(__uint_as_float(b0 << 16)) * f;
                const float y1 = fabsf(__uint_as_float(b1 << 16)) * f;
                uint32_t pair = cvt_e4m3x2(y0, y1);
                pair |= ((b0 >> 15) & 1u) << 7;
                pair |= ((b1 >> 15) & 1u) << 15;
                word |= pair << (8 * e);
            }
            words[gi][q] = word;
        }
    }
    __syncthreads();  // every read of the bf16 staging is done before it is overwritten
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
        const int g = g0 + 2 * gi;
        uint4 *dst = reinterpret_cast<uint4 *>(&ctile[c * kCPitch + g * 32]);
        dst[0] = make_uint4(words[gi][0], words[gi][1], words[gi][2], words[gi][3]);
        dst[1] = make_uint4(words[gi][4], words[gi][5], words[gi][6], words[gi][7]);
        atom[(c & 31) * 16 + (c >> 5) * 4 + g] = static_cast<uint8_t>(Xs[gi] + 127);
    }
    __syncthreads();
    const int64_t head = static_cast<int64_t>(b) * H + h;
    for (int i = threadIdx.x; i < 128 * 8; i += 256) {
        const int row = i >> 3, ch = i & 7;
        *reinterpret_cast<uint4 *>(codes + (head * 128 + row) * cap + t0 + ch * 16) =
            *reinterpret_cast<const uint4 *>(&ctile[row * kCPitch + ch * 16]);
    }
    if (threadIdx.x < 32)
        reinterpret_cast<uint4 *>(scales + (head * nblk + blk) * 512)[threadIdx.x] =
            reinterpret_cast<const uint4 *>(atom)[threadIdx.x];
}

cudaError_t launch_quantize_qk(const void *x, int B, int S, int H, int64_t sb, int64_t ss, int64_t sh,
                               const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                               cudaStream_t stream, bool pad_to_cap) {
    const int row_len = pad_to_cap ? cap : S;
    const int64_t rows = static_cast<int64_t>(B) * row_len * H;
    const int rows_per_cta = 256 / 16;
    int64_t grid = (rows + rows_per_cta - 1) / rows_per_cta;
    const int64_t max_grid = 148 * 16;
    if (grid > max_grid) grid = max_grid;
    if (grid < 1) grid = 1;
    quantize_qk_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(x), B, S, H, sb, ss, sh, seqlens, cap, row_len, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_quantize_v(const void *v, int B, int S, int H, int64_t sb, int64_t ss, int64_t sh,
                              const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                              cudaStream_t stream) {
    const int64_t grid = static_cast<int64_t>(B) * H * (cap / 128);
    quantize_v_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(v), B, S, H, sb, ss, sh, seqlens, cap, codes, scales);
    return cudaGetLastError();
}

}  // namespace qk4v8
