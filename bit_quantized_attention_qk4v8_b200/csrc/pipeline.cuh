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

// A warp's copy of 32 consecutive block-table entries of one sequence.
struct PageLookup {
    int b = -1, base = 0, entry = 0;
};

// Where key tile `tile` of (b, h_kv) lives: `row` of the [rows][tokens] K/V
// tensor maps and scale arrays, and the 128-token block `blk` in that row.
// Contiguous cache: row b * Hkv + h_kv, block `tile`. Paged cache: page
// block_table[b][tile], row page * Hkv + h_kv, block 0; the warp loads the
// entries 32 tiles at a time. An entry outside [0, num_pages) reads page 0
// instead and records QK4V8_ERR_INVALID_ARG (1) in *status. All 32 lanes of
// the warp call it with the same arguments. kPaging = false compiles the
// contiguous case alone (kernel instances that never see a block table).
template <bool kPaging>
__device__ __forceinline__ void kv_tile_row(const AttnParams &p, int b, int h_kv, int tile, PageLookup &pl, int &row,
                                            int &blk) {
    if (!kPaging || !p.block_table) {
        row = b * p.Hkv + h_kv;
        blk = tile;
        return;
    }
    const int base = tile & ~31;
    if (pl.b != b || pl.base != base) {
        const int t = base + static_cast<int>(threadIdx.x & 31);
        pl.entry = t < p.max_pages ? p.block_table[static_cast<int64_t>(b) * p.max_pages + t] : 0;
        pl.b = b;
        pl.base = base;
    }
    int page = __shfl_sync(0xffffffffu, pl.entry, tile & 31);
    if (page < 0 || page >= p.num_pages) {
        if ((threadIdx.x & 31) == 0 && p.status) atomicCAS(p.status, 0, 1);
        page = 0;
    }
    row = page * p.Hkv + h_kv;
    blk = 0;
}

// 128-token blocks per row of the K/V scale arrays.
template <bool kPaging>
__device__ __forceinline__ int kv_row_blocks(const AttnParams &p) {
    return kPaging && p.block_table ? 1 : p.kv_cap / 128;
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
