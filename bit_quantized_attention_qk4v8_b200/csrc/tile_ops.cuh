// Small per-thread helpers shared by the kernels whose softmax threads own
// one query row of a TMEM accumulator (the prefill kernel and the GQA decode
// kernel): row maxima over raw score registers, narrow TMEM loads and stores,
// shared-space stores, the bounded peer wait, the in-place O rescale and the
// end-of-CTA TMEM release.
#pragma once

#include <cstdint>

#include "pipeline.cuh"
#include "ptx.cuh"

namespace qk4v8 {

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Largest of 32 floats (as raw bits), a tree of three-input maxima.
__device__ __forceinline__ float max32(const uint32_t (&s)[32]) {
    float t[11];
#pragma unroll
    for (int g = 0; g < 10; ++g)
        t[g] = fmax3(__uint_as_float(s[3 * g]), __uint_as_float(s[3 * g + 1]), __uint_as_float(s[3 * g + 2]));
    t[10] = fmaxf(__uint_as_float(s[30]), __uint_as_float(s[31]));
    const float a = fmax3(t[0], t[1], t[2]), b = fmax3(t[3], t[4], t[5]), c = fmax3(t[6], t[7], t[8]);
    return fmaxf(fmax3(a, b, c), fmaxf(t[9], t[10]));
}

__device__ __forceinline__ uint32_t tc_ld_32x32b_x1(uint32_t taddr) {
    uint32_t r;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
    return r;
}

__device__ __forceinline__ void tc_ld_32x32b_x4(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}

__device__ __forceinline__ void tc_st_32x32b_x4(uint32_t taddr, const uint32_t (&r)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t a) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// Wait on an mbarrier phase that every peer reaches within its own bounded
// waits. It does not give up on the abort flag, so all waiters see the same
// phase and take the same branch afterwards.
constexpr uint64_t kPeerWaitTimeoutNs = 4 * kWaitTimeoutNs;

static __device__ __noinline__ bool wait_peers_slow(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 20000))
        if (globaltimer_ns() - t0 > kPeerWaitTimeoutNs) return false;
    return true;
}

__device__ __forceinline__ bool wait_peers(uint64_t *bar, uint32_t parity) {
    return mbar_try_wait(bar, parity) || wait_peers_slow(bar, parity);
}

// O *= 2^-E for `ncols` columns (a multiple of 4) at taddr of this thread's
// TMEM lane, E >= 0.
static __device__ __noinline__ void rescale_o_lane(uint32_t taddr, int ncols, int E) {
    const float a = E < 126 ? __uint_as_float(static_cast<uint32_t>(127 - E) << 23) : 0.f;
    for (int c = 0; c < ncols; c += 4) {
        uint32_t o[4];
        tc_ld_32x32b_x4(taddr + c, o);
        tc_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * a);
        tc_st_32x32b_x4(taddr + c, o);
    }
    tc_wait_st();
}

// End of the CTA: every warp arrives here from its own role branch (the role
// branches hold different live registers, so they never share this code); the
// warp that allocated the tensor memory then frees it.
__device__ __forceinline__ void teardown_tmem(bool alloc_warp, uint32_t tmem, uint32_t ncols) {
    tc_fence_before();
    __syncthreads();
    if (alloc_warp) {
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

}  // namespace qk4v8
