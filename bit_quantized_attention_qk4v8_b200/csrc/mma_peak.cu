// Tensor-pipe peak of the block-scaled MMA shapes the attention kernels issue,
// measured with the same instructions and nothing else: each CTA issues a long
// run of tcgen05.mma into one TMEM accumulator from operands resident in shared
// memory (no loads, no softmax). Used as the denominator of the prefill
// roofline; it is a measurement aid, not part of the attention path.
#include <cuda_runtime.h>

#include <cstdint>

#include "pipeline.cuh"
#include "ptx.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

namespace {

constexpr int kMpThreads = 128;
constexpr int kMpA = 0;               // A: 128 rows x 128 B (128-byte swizzle)
constexpr int kMpB = 128 * 128;       // B: up to 256 rows x 128 B
constexpr int kMpSf = kMpB + 256 * 128;  // 512-byte scale atom, all 2^0
constexpr int kMpBar = kMpSf + 512;
constexpr int kMpBytes = kMpBar + 64 + 1024;

constexpr uint32_t mp_idesc(uint32_t fmt, uint32_t n) {
    return (fmt << 7) | (fmt << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}

}  // namespace

// kind: 0 = mxf4 (E2M1) N=128 K=64, 1 = mxf8f6f4 (E4M3) N=144 K=32,
//       2 = mxf8f6f4 N=256 K=32, 3 = mxf4 N=256 K=64.
__global__ void __launch_bounds__(kMpThreads, 1) qk4v8_mma_peak_kernel(int kind, int iters, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *done = reinterpret_cast<uint64_t *>(smem + kMpBar);
    uint32_t *slot = reinterpret_cast<uint32_t *>(smem + kMpBar + 8);
    // Operands: a fixed pseudo-random byte pattern (the tensor pipe's rate does
    // not depend on values, but all-zero data would draw less power).
    for (int i = threadIdx.x; i < kMpSf / 4; i += kMpThreads)
        reinterpret_cast<uint32_t *>(smem)[i] = (0x9E3779B9u * (i + 1)) & 0x3B3B3B3Bu;
    for (int i = threadIdx.x; i < 128; i += kMpThreads) reinterpret_cast<uint32_t *>(smem + kMpSf)[i] = 0x7F7F7F7Fu;
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_barrier_init();
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    if (warp == 0) {
        if (lane == 0) {
            const uint32_t sb = smem_u32(smem);
            const uint32_t tSfA = tmem + 400, tSfB = tmem + 404;
            const uint64_t dSf = smem_desc(sb + kMpSf, 0, 128, 0);
            tc_cp_32x128b_warpx4(tSfA, dSf);
            tc_cp_32x128b_warpx4(tSfB, dSf);
            tc_cp_32x128b_warpx4(tSfB + 4, dSf);
            const bool fp4 = kind == 0 || kind == 3;
            const uint32_t n = kind == 0 ? 128u : (kind == 1 ? 144u : 256u);
            const uint32_t idesc = mp_idesc(fp4 ? 1u : 0u, n);
            const uint64_t dA = smem_desc(sb + kMpA, 16, 1024, 2);
            const uint64_t dB = smem_desc(sb + kMpB, 16, 1024, 2);
            for (int i = 0; i < iters; ++i) {
                const uint32_t k = static_cast<uint32_t>(i & 3);
                if (fp4)
                    tc_mma_mxf4(tmem, dA + 2 * (k & 1), dB + 2 * (k & 1), idesc | ((2 * (k & 1)) << 29) | ((2 * (k & 1)) << 4),
                                tSfA | ((2 * (k & 1)) << 30), tSfB | ((2 * (k & 1)) << 30), i > 0 ? 1u : 0u);
                else
                    tc_mma_mxf8(tmem, dA + 2 * k, dB + 2 * k, idesc | (k << 29) | (k << 4), tSfA | (k << 30),
                                tSfB | (k << 30), i > 0 ? 1u : 0u);
            }
            tc_commit(done);
        }
        __syncwarp();
        // Bounded wait for the run to drain before TMEM is freed.
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(done, 0, 100000))
            if (globaltimer_ns() - t0 > 4 * kWaitTimeoutNs) {
                if (status && lane == 0) atomicCAS(status, 0, 4);
                break;
            }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

cudaError_t launch_mma_peak(int kind, int ctas, int iters, int32_t *status, cudaStream_t stream) {
    constexpr int kMaxDevices = 64;
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !configured[dev]) {
        e = cudaFuncSetAttribute(qk4v8_mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMpBytes);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) configured[dev] = true;
    }
    qk4v8_mma_peak_kernel<<<ctas, kMpThreads, kMpBytes, stream>>>(kind, iters, status);
    return cudaGetLastError();
}

}  // namespace qk4v8
