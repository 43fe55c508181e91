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

}  // namespace qk4v8
