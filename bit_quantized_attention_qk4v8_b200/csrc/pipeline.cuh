// Pipeline helpers shared by the attention kernels: bounded mbarrier waits,
// named-barrier votes and small integer helpers.
#pragma once

#include <cstdint>

#include "ptx.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

__device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }
__device__ __forceinline__ int imax(int a, int b) { return a > b ? a : b; }

// First key a decode query block of a sequence of L keys may see: with a
// window, the last `window` keys before the block's Sq tokens (MiMo DFlash
// article, section on block-diffusion speculative decoding: the draft block
// attends to a sliding window over the most recent context), else key 0.
__device__ __forceinline__ int kv_window_lo(const AttnParams &p, int L) {
    return p.window > 0 ? imax(0, L - p.Sq - p.window) : 0;
}

__device__ __forceinline__ bool aborted(volatile uint32_t *flag, const int32_t *status) {
    if (*flag) return true;
    if (status && *reinterpret_cast<const volatile int32_t *>(status) != 0) {
        *flag = 1;
        return true;
    }
    return false;
}

// Bounded wait on an mbarrier phase. Each try sleeps in hardware for up to
// kWaitSleepNs. When the total wait exceeds kWaitTimeoutNs, it records
// QK4V8_ERR_TIMEOUT (4) in *status and raises the CTA abort flag. Once the flag
// is up, or another CTA has reported a status, every wait returns false
// promptly, so the CTA unwinds instead of hanging.
constexpr uint32_t kWaitSleepNs = 200000;

static __device__ __noinline__ bool wait_bar_slow(uint64_t *bar, uint32_t parity, volatile uint32_t *flag,
                                                  int32_t *status) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
        if (aborted(flag, status)) return false;
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
            *flag = 1;
            if (status) atomicCAS(status, 0, 4);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile uint32_t *flag, int32_t *status) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    return wait_bar_slow(bar, parity, flag, status);
}

// Named barrier over `nthreads` threads that also ORs a predicate across them.
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
        : "memory");
    return out != 0;
}

__device__ __forceinline__ void bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Float max over the warp through an order-preserving integer key.
__device__ __forceinline__ float warp_max_f32(float x) {
    int k = __float_as_int(x);
    k = k >= 0 ? k : (k ^ 0x7FFFFFFF);
    k = __reduce_max_sync(0xffffffffu, k);
    k = k >= 0 ? k : (k ^ 0x7FFFFFFF);
    return __int_as_float(k);
}

__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace qk4v8
