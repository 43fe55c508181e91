// MX element encoders shared by the quantization kernels and the decode
// kernel's in-kernel query quantization, so both produce identical bytes.
//
// Scale rule (OCP MX, as the MpFA QK4V8 article applies it in sections
// 2.1-2.2 and 3.2): one E8M0 scale 2^X per block of 32 values, with
// X = floor(log2 amax) - emax, clamped to [-127, 127]; each element is the
// nearest code of x / 2^X, ties to even, saturating at the format's maximum.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace qk4v8 {

// Shared exponent from the float bits of a non-negative amax.
// floor(log2 amax) is the unbiased exponent field; bf16 inputs that are
// subnormal (or zero) land at the -127 clamp for both element formats.
__device__ __forceinline__ int shared_exponent(float amax, int emax) {
    int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF);
    int X = e - 127 - emax;
    X = X < -127 ? -127 : X;
    X = X > 127 ? 127 : X;
    return X;
}

__device__ __forceinline__ float pow2_neg(int X) {  // 2^-X for X in [-127, 126]
    return __uint_as_float(static_cast<uint32_t>(127 - X) << 23);
}

// MXFP4 encode of eight consecutive channels of a 128-channel row held by 16
// lanes (lane sub = lane & 15 holds channels 8 sub .. 8 sub + 7, so four
// lanes share one block of 32). All 32 lanes of the warp must call it
// together. Returns the eight E2M1 codes packed two per byte (even channel in
// the low nibble, the input's sign bit kept) and sets X to the block's shared
// exponent; an invalid row encodes as zero codes.
__device__ __forceinline__ uint32_t mxfp4_encode8(uint4 raw, bool valid, int &X) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    float v[8];
    float amax = 0.f;
    uint32_t sign = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        sign |= ((w[i] >> 15) & 1u) << (8 * i + 3);
        sign |= ((w[i] >> 31) & 1u) << (8 * i + 7);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    X = shared_exponent(amax, 2);
    const float f = pow2_neg(X);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fabsf(v[i]) * f;  // exact: power-of-two scaling
    return valid ? (cvt_e2m1x8(v) | sign) : 0u;
}

// MXFP4 encode of eight fp32 values (the rotated rows), same lane layout and
// contract as mxfp4_encode8; the sign of each code is the sign bit of the
// float.
__device__ __forceinline__ uint32_t mxfp4_encode8_f32(const float (&x)[8], bool valid, int &X) {
    float v[8];
    float amax = 0.f;
    uint32_t sign = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        sign |= (__float_as_uint(x[i]) >> 31) << (4 * i + 3);
        amax = fmaxf(amax, fabsf(x[i]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    X = shared_exponent(amax, 2);
    const float f = pow2_neg(X);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fabsf(x[i]) * f;  // exact: power-of-two scaling
    return valid ? (cvt_e2m1x8(v) | sign) : 0u;
}

// Rotation of a 128-channel row by H / sqrt(128), H the Sylvester Hadamard
// matrix (MpFA article, sections 2.1 and 3.1: a light rotation before the
// 4-bit quantization spreads outlier channels over the row). The row is held
// by 16 lanes, 8 consecutive channels each (lane sub = lane & 15 holds
// channels 8 sub .. 8 sub + 7). Fast Walsh-Hadamard transform in fp32:
// butterfly stages of stride 1, 2 and 4 inside the lane, then 8, 16, 32 and 64
// across lanes (lane xor 1, 2, 4, 8); each stage maps the pair (a, b) at
// channels (i, i + stride) to (a + b, a - b). Then one multiply by the fp32
// value nearest 2^-3.5. All 32 lanes of the warp must call it together.
__device__ __forceinline__ void hadamard128_rows(float (&v)[8], int sub) {
#pragma unroll
    for (int s = 1; s < 8; s *= 2) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i & s) continue;
            const float a = v[i], b = v[i + s];
            v[i] = a + b;
            v[i + s] = a - b;
        }
    }
#pragma unroll
    for (int m = 1; m < 16; m *= 2) {
        const bool upper = (sub & m) != 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float other = __shfl_xor_sync(0xffffffffu, v[i], m);
            v[i] = upper ? other - v[i] : v[i] + other;
        }
    }
    constexpr float kRsqrt128 = 0x1.6a09e6p-4f;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = v[i] * kRsqrt128;
}

}  // namespace qk4v8
