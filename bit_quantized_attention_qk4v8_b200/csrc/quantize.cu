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

// One lane per MX group: 4 lanes per 128-channel (token, head) row, 32
// channels (64 bytes of bf16) per lane, so the group amax needs no shuffle and
// a warp takes 8 rows per step. blockIdx.y is the batch entry; its rows (t, h)
// are visited in input order (t major), so a warp's loads are contiguous.
// Tokens 0 .. row_len-1 of each sequence are visited: row_len = cap writes the
// whole capacity (zero codes and scales past the valid length), row_len = S
// only the rows of the input. Each lane steps its (t, h) position by a fixed
// amount: an integer division per row would make the kernel bound by
// instruction issue instead of memory.
//
// With kRotate the row is first rotated by H / sqrt(128), H the Sylvester
// Hadamard matrix (MpFA article, sections 2.1 and 3.1), in fp32 as the fast
// Walsh-Hadamard transform: butterfly stages of stride 1..16 inside the lane,
// 32 and 64 across the row's lanes (lane xor 1, 2), each mapping the pair
// (a, b) at channels (i, i + stride) to (a + b, a - b); then one multiply by
// the fp32 value nearest 2^-3.5. Packed f32x2 adds give the same bits as
// scalar ones.

// Butterfly stage of stride s (s >= 2) over a lane's 32 values held as 16 pairs.
template <int S>
__device__ __forceinline__ void fwht_stage_pairs(float2 (&w)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if ((2 * i) & S) continue;
        const float2 a = w[i], b = w[i + S / 2];
        w[i] = fadd2(a, b);
        w[i + S / 2] = fsub2(a, b);
    }
}

// Rows of batch entry b taken by CTA bx of the gx CTAs that share the entry
// (the body of quantize_qk_kernel, also run by quantize_qkv_kernel).
template <bool kRotate>
__device__ __forceinline__ void qk_rows(const __nv_bfloat16 *__restrict__ x, int S, int H, int64_t sb, int64_t ss,
                                        int64_t sh, const int32_t *__restrict__ seqlens, int cap, int row_len,
                                        uint8_t *__restrict__ codes, uint8_t *__restrict__ scales, int b, int bx,
                                        int gx) {
    const int lane = threadIdx.x & 31;
    const int g = lane & 3;   // MX group (channels 32g .. 32g+31) of this lane
    const int rows = row_len * H;  // rows of this batch entry (the launcher keeps this below 2^30)
    int valid_len = S;
    if (seqlens) {
        const int L = seqlens[b];
        valid_len = L < valid_len ? L : valid_len;
    }
    const int step = gx * (blockDim.x >> 5) * 8;  // rows per grid step
    const int step_t = step / H, step_h = step - step_t * H;
    // The loop bound is taken per warp (8 rows) so every lane reaches the shuffles.
    int base = (bx * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 8;
    int t = (base + (lane >> 2)) / H;
    int h = (base + (lane >> 2)) - t * H;
    const __nv_bfloat16 *xb = x + b * sb;
    const int64_t head_b = static_cast<int64_t>(b) * H;
    const int nblk = cap / 128;
    for (; base < rows; base += step) {
        const bool in = base + (lane >> 2) < rows;
        const bool valid = in && t < valid_len;
        uint4 raw[4] = {};
        if (valid) {
            const uint4 *src = reinterpret_cast<const uint4 *>(xb + t * ss + h * sh + g * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) raw[i] = src[i];
        }
        // bf16 -> f32, exact: channel 2k in the low half of word k.
        float2 w[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t ws[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
                w[4 * i + k] = make_float2(__uint_as_float(ws[k] << 16), __uint_as_float(ws[k] & 0xFFFF0000u));
        }
        if (kRotate) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {  // stride 1: the two halves of each pair
                const float a = w[i].x, c = w[i].y;
                w[i] = make_float2(a + c, a - c);
            }
            fwht_stage_pairs<2>(w);
            fwht_stage_pairs<4>(w);
            fwht_stage_pairs<8>(w);
            fwht_stage_pairs<16>(w);
#pragma unroll
            for (int m = 1; m <= 2; m <<= 1) {  // strides 32 and 64: the row's other lanes
                // The upper lane keeps o - w, the lower one w + o: one fused
                // s * w + o with s = -1 or +1, which rounds exactly as the
                // subtraction or the addition does.
                const float s = (g & m) != 0 ? -1.f : 1.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, w[i].x, m),
                                                 __shfl_xor_sync(0xffffffffu, w[i].y, m));
                    w[i] = ffma2(make_float2(s, s), w[i], o);
                }
            }
            constexpr float kRsqrt128 = 0x1.6a09e6p-4f;
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = fmul2(w[i], make_float2(kRsqrt128, kRsqrt128));
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(w[i].x), fabsf(w[i].y)));
        const int X = shared_exponent(amax, 2);
        const float f = pow2_neg(X);
        // x / 2^X is exact (power-of-two scaling); the conversion rounds the
        // magnitude and keeps the sign bit, also of a value that rounds to zero.
        uint32_t packed[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 a = fmul2(w[4 * q + e], make_float2(f, f));
                y[2 * e] = a.x;
                y[2 * e + 1] = a.y;
            }
            packed[q] = valid ? cvt_e2m1x8(y) : 0u;
        }
        if (in) {
            *reinterpret_cast<uint4 *>(codes + ((head_b + h) * cap + t) * 64 + g * 16) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
            scales[((head_b + h) * nblk + t / 128) * 512 + (t & 31) * 16 + ((t & 127) >> 5) * 4 + g] =
                valid ? static_cast<uint8_t>(X + 127) : 0;
        }
        t += step_t;
        h += step_h;
        if (h >= H) {
            h -= H;
            ++t;
        }
    }
}

template <bool kRotate>
__global__ void __launch_bounds__(256, kRotate ? 3 : 4) quantize_qk_kernel(const __nv_bfloat16 *__restrict__ x, int S,
                                                                           int H, int64_t sb, int64_t ss, int64_t sh,
                                                                           const int32_t *__restrict__ seqlens,
                                                                           int cap, int row_len,
                                                                           uint8_t *__restrict__ codes,
                                                                           uint8_t *__restrict__ scales) {
    qk_rows<kRotate>(x, S, H, sb, ss, sh, seqlens, cap, row_len, codes, scales, static_cast<int>(blockIdx.y),
                     static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
}

// ------------------------------------------------------------------ MXFP8 V

// One CTA per (b, h, 128-token block): stage the bf16 tile in shared memory,
// quantize each channel's four 32-token groups, and write the block's codes
// (128 channel rows of 128 tokens, 16 KiB contiguous) plus its 512-byte scale
// atom.
constexpr int kVPitch = 136;  // bf16 elements per staged token row (16-byte padding)
constexpr int kCPitch = 144;  // bytes per staged code row

// Loads the bf16 tile of 128 tokens x 128 channels of (b, h) from token t0 into
// shared memory (row pitch kVPitch): all eight 16-byte loads of a thread are
// issued before the first store, so a CTA keeps its whole 32 KiB in flight.
// Tokens at or past valid_len read as zeros. Ends with a CTA barrier.
__device__ __forceinline__ void stage_v_tile(const __nv_bfloat16 *__restrict__ v, int b, int h, int t0,
                                             int valid_len, int64_t sb, int64_t ss, int64_t sh,
                                             uint16_t *tile) {
    uint4 raw[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int i = threadIdx.x + 256 * k;
        const int tk = i >> 4, ch = i & 15;
        raw[k] = make_uint4(0, 0, 0, 0);
        if (t0 + tk < valid_len)
            raw[k] = *reinterpret_cast<const uint4 *>(v + b * sb + static_cast<int64_t>(t0 + tk) * ss + h * sh +
                                                      ch * 8);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int i = threadIdx.x + 256 * k;
        *reinterpret_cast<uint4 *>(&tile[(i >> 4) * kVPitch + (i & 15) * 8]) = raw[k];
    }
    __syncthreads();
}

// Encoder thread layout of both V kernels: thread (cp, g) = (threadIdx.x & 63,
// threadIdx.x >> 6) takes channels 2cp and 2cp + 1 over the 32 tokens of group
// g. One 32-bit shared load per token gives both channels (a warp reads 128
// contiguous bytes of a staged row), and the registers then serve the amax and
// the encode. The amax of both channels is one bf16x2 max chain: max is exact
// in bf16, so it equals the fp32 amax.
__device__ __forceinline__ void load_v_pair(const uint16_t *tile, int cp, int g, int emax, uint32_t (&w)[32],
                                            int (&X)[2]) {
    const uint32_t *t32 = reinterpret_cast<const uint32_t *>(tile);
    __nv_bfloat162 m = __floats2bfloat162_rn(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        w[j] = t32[(g * 32 + j) * (kVPitch / 2) + cp];
        m = __hmax2(m, __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j])));
    }
    const uint32_t mb = *reinterpret_cast<const uint32_t *>(&m);
    X[0] = shared_exponent(__uint_as_float(mb << 16), emax);
    X[1] = shared_exponent(__uint_as_float(mb & 0xFFFF0000u), emax);
}

// bf16 channel k (0: low half, 1: high half) of a staged word as fp32, exact.
__device__ __forceinline__ float v_chan(uint32_t w, int k) {
    return __uint_as_float(k ? (w & 0xFFFF0000u) : (w << 16));
}

// Staged code rows: channel 2cp at row cp, channel 2cp + 1 at row 64 + cp, so
// the 32 threads of a warp store to consecutive rows.
__device__ __forceinline__ int v_code_row(int channel) { return (channel >> 1) + (channel & 1) * 64; }

// Tile `idx` = (b, h, 128-token block) of V (the body of quantize_v_kernel,
// also run by quantize_qkv_kernel).
__device__ __forceinline__ void v_tile(const __nv_bfloat16 *__restrict__ v, int S, int H, int64_t sb, int64_t ss,
                                       int64_t sh, const int32_t *__restrict__ seqlens, int cap,
                                       uint8_t *__restrict__ codes, uint8_t *__restrict__ scales, int idx) {
    __shared__ __align__(16) uint16_t tile[128 * kVPitch];  // bf16 staging, later the code tile
    __shared__ __align__(16) uint8_t atom[512];
    uint8_t *ctile = reinterpret_cast<uint8_t *>(tile);     // [128 code rows][kCPitch] after the barrier
    const int nblk = cap / 128;
    const int blk = idx % nblk;
    const int h = (idx / nblk) % H;
    const int b = idx / (nblk * H);
    const int t0 = blk * 128;
    int valid_len = S;
    if (seqlens) {
        int L = seqlens[b];
        valid_len = L < valid_len ? L : valid_len;
    }
    // Stage: invalid tokens read as zeros, which leaves them out of every amax
    // and gives them code 0; a group with no valid token gets scale byte 0.
    stage_v_tile(v, b, h, t0, valid_len, sb, ss, sh, tile);
    const int cp = threadIdx.x & 63;
    const int g = threadIdx.x >> 6;
    uint32_t w[32];
    int X[2];
    load_v_pair(tile, cp, g, 8, w, X);
    // x / 2^X is exact (power-of-two scaling); the conversion rounds the
    // magnitude and keeps the sign bit, also of a value that rounds to zero.
    uint32_t words[2][8];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float f = pow2_neg(X[k]);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const uint32_t a = cvt_e4m3x2(v_chan(w[4 * q], k) * f, v_chan(w[4 * q + 1], k) * f);
            const uint32_t c = cvt_e4m3x2(v_chan(w[4 * q + 2], k) * f, v_chan(w[4 * q + 3], k) * f);
            words[k][q] = a | (c << 16);
        }
    }
    __syncthreads();  // every read of the bf16 staging is done before it is overwritten
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int c = 2 * cp + k;
        uint4 *dst = reinterpret_cast<uint4 *>(&ctile[v_code_row(c) * kCPitch + g * 32]);
        dst[0] = make_uint4(words[k][0], words[k][1], words[k][2], words[k][3]);
        dst[1] = make_uint4(words[k][4], words[k][5], words[k][6], words[k][7]);
        atom[(c & 31) * 16 + (c >> 5) * 4 + g] = static_cast<uint8_t>(X[k] + 127);
    }
    __syncthreads();
    const int64_t head = static_cast<int64_t>(b) * H + h;
    uint8_t *block = codes + (head * nblk + blk) * (128 * 128);  // the tile's 16 KiB, channel rows of 128 B
    for (int i = threadIdx.x; i < 128 * 8; i += 256) {
        const int row = i >> 3, ch = i & 7;
        *reinterpret_cast<uint4 *>(block + row * 128 + ch * 16) =
            *reinterpret_cast<const uint4 *>(&ctile[v_code_row(row) * kCPitch + ch * 16]);
    }
    if (threadIdx.x < 32)
        reinterpret_cast<uint4 *>(scales + (head * nblk + blk) * 512)[threadIdx.x] =
            reinterpret_cast<const uint4 *>(atom)[threadIdx.x];
}

__global__ void __launch_bounds__(256, 5) quantize_v_kernel(const __nv_bfloat16 *__restrict__ v, int S, int H,
                                                         int64_t sb, int64_t ss, int64_t sh,
                                                         const int32_t *__restrict__ seqlens, int cap,
                                                         uint8_t *__restrict__ codes,
                                                         uint8_t *__restrict__ scales) {
    v_tile(v, S, H, sb, ss, sh, seqlens, cap, codes, scales, static_cast<int>(blockIdx.x));
}

// ------------------------------------------------------------------ Q, K and V in one launch

// CTAs [0, nq) quantize Q (gxq per batch entry), [nq, nq + nk) K (gxk per
// entry), the rest V (one per (b, h, 128-token block)). Small prefills are
// launch-bound: one launch instead of three. Every CTA carries the V staging
// buffer (35 KB), which still allows the four CTAs per SM the registers allow.
struct QkvArgs {
    const __nv_bfloat16 *q, *k, *v;
    int Sq, Sk, Hq, Hkv, q_cap, kv_cap;
    int64_t qsb, qss, qsh, ksb, kss, ksh;
    const int32_t *seqlens_k;
    uint8_t *q_codes, *q_scales, *k_codes, *k_scales, *v_codes, *v_scales;
    int gxq, gxk, nq, nk;
};

__global__ void __launch_bounds__(256, 4) quantize_qkv_kernel(const QkvArgs a) {
    int i = static_cast<int>(blockIdx.x);
    if (i < a.nq) {
        qk_rows<false>(a.q, a.Sq, a.Hq, a.qsb, a.qss, a.qsh, nullptr, a.q_cap, a.q_cap, a.q_codes, a.q_scales,
                       i / a.gxq, i % a.gxq, a.gxq);
        return;
    }
    i -= a.nq;
    if (i < a.nk) {
        qk_rows<false>(a.k, a.Sk, a.Hkv, a.ksb, a.kss, a.ksh, a.seqlens_k, a.kv_cap, a.kv_cap, a.k_codes,
                       a.k_scales, i / a.gxk, i % a.gxk, a.gxk);
        return;
    }
    i -= a.nk;
    v_tile(a.v, a.Sk, a.Hkv, a.ksb, a.kss, a.ksh, a.seqlens_k, a.kv_cap, a.v_codes, a.v_scales, i);
}

// ------------------------------------------------------------------ MXFP4 V

// The QK4V4 comparison point (MpFA article, sections 2.2 and 5.3): V in MXFP4,
// groups of 32 along the token axis like the MXFP8 V. Same staging as
// quantize_v_kernel; each thread encodes the 32-token group of two channels to
// 16 bytes of packed E2M1 each (even token in the low nibble), and the
// 128-token block of a channel row is 64 bytes of codes [B][H][cap / 128][128][64].
constexpr int kC4Pitch = 80;  // bytes per staged code row (64 + 16 padding)

__global__ void __launch_bounds__(256) quantize_v4_kernel(const __nv_bfloat16 *__restrict__ v, int B, int S, int H,
                                                          int64_t sb, int64_t ss, int64_t sh,
                                                          const int32_t *__restrict__ seqlens, int cap,
                                                          uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ scales) {
    __shared__ __align__(16) uint16_t tile[128 * kVPitch];
    __shared__ __align__(16) uint8_t atom[512];
    uint8_t *ctile = reinterpret_cast<uint8_t *>(tile);  // [128 code rows][kC4Pitch] after the barrier
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
    stage_v_tile(v, b, h, t0, valid_len, sb, ss, sh, tile);
    const int cp = threadIdx.x & 63;
    const int g = threadIdx.x >> 6;
    uint32_t w[32];
    int X[2];
    load_v_pair(tile, cp, g, 2, w, X);
    uint32_t words[2][4];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float f = pow2_neg(X[k]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = v_chan(w[8 * q + e], k) * f;
            words[k][q] = cvt_e2m1x8(y);
        }
    }
    __syncthreads();  // every read of the bf16 staging is done before it is overwritten
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int c = 2 * cp + k;
        *reinterpret_cast<uint4 *>(&ctile[v_code_row(c) * kC4Pitch + g * 16]) =
            make_uint4(words[k][0], words[k][1], words[k][2], words[k][3]);
        atom[(c & 31) * 16 + (c >> 5) * 4 + g] = static_cast<uint8_t>(X[k] + 127);
    }
    __syncthreads();
    const int64_t head = static_cast<int64_t>(b) * H + h;
    uint8_t *block = codes + (head * nblk + blk) * (128 * 64);  // the tile's 8 KiB, channel rows of 64 B
    for (int i = threadIdx.x; i < 128 * 4; i += 256) {
        const int row = i >> 2, ch = i & 3;
        *reinterpret_cast<uint4 *>(block + row * 64 + ch * 16) =
            *reinterpret_cast<const uint4 *>(&ctile[v_code_row(row) * kC4Pitch + ch * 16]);
    }
    if (threadIdx.x < 32)
        reinterpret_cast<uint4 *>(scales + (head * nblk + blk) * 512)[threadIdx.x] =
            reinterpret_cast<const uint4 *>(atom)[threadIdx.x];
}

cudaError_t launch_quantize_v4(const void *v, int B, int S, int H, int64_t sb, int64_t ss, int64_t sh,
                               const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                               cudaStream_t stream) {
    const int64_t grid = static_cast<int64_t>(B) * H * (cap / 128);
    quantize_v4_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(v), B, S, H, sb, ss, sh, seqlens, cap, codes, scales);
    return cudaGetLastError();
}

// CTAs per batch entry of the Q/K part: about one wave over all entries (4 CTAs
// per SM, 3 with the rotation), 64 rows per CTA per step.
static int64_t qk_ctas_per_entry(int64_t rows, int B, bool rotate) {
    int64_t gx = (rows + 63) / 64;
    const int64_t wave = (148 * (rotate ? 3 : 4) + B - 1) / B;
    if (gx > wave) gx = wave;
    return gx < 1 ? 1 : gx;
}

cudaError_t launch_quantize_qk(const void *x, int B, int S, int H, int64_t sb, int64_t ss, int64_t sh,
                               const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                               cudaStream_t stream, bool pad_to_cap, bool rotate) {
    const int row_len = pad_to_cap ? cap : S;
    const int64_t rows = static_cast<int64_t>(row_len) * H;  // per batch entry
    if (rows >= (int64_t{1} << 30)) return cudaErrorInvalidValue;
    const int64_t gx = qk_ctas_per_entry(rows, B, rotate);
    // The grid's y extent is at most 65535: larger batches go in chunks.
    const int64_t codes_per_b = static_cast<int64_t>(H) * cap * 64;
    const int64_t scales_per_b = static_cast<int64_t>(H) * (cap / 128) * 512;
    for (int b0 = 0; b0 < B; b0 += 65535) {
        const int nb = B - b0 < 65535 ? B - b0 : 65535;
        const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(nb));
        const __nv_bfloat16 *xs = static_cast<const __nv_bfloat16 *>(x) + b0 * sb;
        const int32_t *ls = seqlens ? seqlens + b0 : nullptr;
        if (rotate)
            quantize_qk_kernel<true><<<grid, 256, 0, stream>>>(xs, S, H, sb, ss, sh, ls, cap, row_len,
                                                               codes + b0 * codes_per_b, scales + b0 * scales_per_b);
        else
            quantize_qk_kernel<false><<<grid, 256, 0, stream>>>(xs, S, H, sb, ss, sh, ls, cap, row_len,
                                                                codes + b0 * codes_per_b, scales + b0 * scales_per_b);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_quantize_v(const void *v, int B, int S, int H, int64_t sb, int64_t ss, int64_t sh,
                              const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                              cudaStream_t stream) {
    const int64_t grid = static_cast<int64_t>(B) * H * (cap / 128);
    quantize_v_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(v), S, H, sb, ss, sh, seqlens, cap, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_quantize_qkv(const void *q, const void *k, const void *v, int B, int Sq, int Sk, int Hq, int Hkv,
                                const int32_t *seqlens_k, int q_cap, int kv_cap, uint8_t *q_codes, uint8_t *q_scales,
                                uint8_t *k_codes, uint8_t *k_scales, uint8_t *v_codes, uint8_t *v_scales,
                                cudaStream_t stream) {
    const int64_t rows_q = static_cast<int64_t>(q_cap) * Hq, rows_k = static_cast<int64_t>(kv_cap) * Hkv;
    if (rows_q >= (int64_t{1} << 30) || rows_k >= (int64_t{1} << 30)) return cudaErrorInvalidValue;
    QkvArgs a{};
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k);
    a.v = static_cast<const __nv_bfloat16 *>(v);
    a.Sq = Sq;
    a.Sk = Sk;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.q_cap = q_cap;
    a.kv_cap = kv_cap;
    a.qsh = 128;
    a.qss = static_cast<int64_t>(Hq) * 128;
    a.qsb = a.qss * Sq;
    a.ksh = 128;
    a.kss = static_cast<int64_t>(Hkv) * 128;
    a.ksb = a.kss * Sk;
    a.seqlens_k = seqlens_k;
    a.q_codes = q_codes;
    a.q_scales = q_scales;
    a.k_codes = k_codes;
    a.k_scales = k_scales;
    a.v_codes = v_codes;
    a.v_scales = v_scales;
    a.gxq = static_cast<int>(qk_ctas_per_entry(rows_q, B, false));
    a.gxk = static_cast<int>(qk_ctas_per_entry(rows_k, B, false));
    const int64_t nq = static_cast<int64_t>(B) * a.gxq, nk = static_cast<int64_t>(B) * a.gxk;
    const int64_t nv = static_cast<int64_t>(B) * Hkv * (kv_cap / 128);
    if (nq + nk + nv >= (int64_t{1} << 31)) return cudaErrorInvalidValue;
    a.nq = static_cast<int>(nq);
    a.nk = static_cast<int>(nk);
    quantize_qkv_kernel<<<static_cast<unsigned>(nq + nk + nv), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace qk4v8
