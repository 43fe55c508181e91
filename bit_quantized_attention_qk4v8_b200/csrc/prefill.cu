// Prefill kernel for QK4V8 attention on sm_100a.
//
// MpFA QK4V8 article (mhpn.cn), sections 2.3, 3.3 and 5.1: attention runs
// block by block with an FP32 online softmax. The 4-bit Q K^T scores are
// dequantized as they come out of the tensor core, and P multiplies the 8-bit
// V into an FP32 accumulator. Both dequantizations are folded into
// block-scaled tcgen05 MMAs:
//   S = Q K^T      kind::mxf4 (E2M1 x E2M1), the E8M0 group scales of Q and K
//                  read from TMEM by the tensor core.
//   O += P V       kind::mxf8f6f4 (E4M3 x E4M3), V's per-channel, per-32-token
//                  scales and one E8M0 scale per (query row, 32-key block) of P.
//
// One CTA computes 128 query rows (one query head, 128 consecutive tokens)
// against the KV head of its GQA group, key tile by key tile (128 keys).
//
// The softmax is spread over 16 warps: warp (cg, quarter) owns TMEM lane
// quarter `quarter` (query rows 32*quarter .. +31) and key block cg (keys
// 32*cg .. +31 of each tile), one query row per thread. Since P carries one
// scale per (row, 32-key block), each thread keeps its own reference max m_w
// for its row and block, with no per-tile exchange:
//   - p = 2^(s*scale - m_w) <= 2^8. m_w moves only when a score passes it by
//     2^8, and then by a whole number of binades.
//   - The O accumulator has one reference m_O per row, agreed by the row's
//     four threads on the first tile (the tile's row max). e = m_w - m_O is an
//     integer held in the block's scale byte.
//   - The block's largest p is brought to [2^7, 2^8) by a further power of
//     two 2^-x, also folded into the scale byte: 127 + e + x.
//   - O is rescaled (rarely) only when some e passes 2^64: the four threads
//     of a row vote, agree on the shift E, scale their share of O's columns by
//     2^-E and lower e by E.
// P is kept as two E4M3 terms with the same scales: P_hi = E4M3(p) and
// P_lo = E4M3(p - P_hi), about 8 significant bits. V carries an extra row of
// ones, so O column 128 accumulates the softmax denominator sum(P_hi + P_lo)
// in the same MMAs.
//
// Warp roles (576 threads): warp 0 TMA producer, warp 1 TMEM allocator and MMA
// issuer, warps 2..17 softmax and epilogue.
//
// kStageQK builds the QK^T stage alone over the same tile schedule: Q/K loads
// with their scales, the mxf4 MMAs and the TMEM drain with the row max. It
// skips exp, P and P V, and writes each row's max scaled score (log2 units)
// to lse instead of an output.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pipeline.cuh"
#include "ptx.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

namespace {

constexpr int kPfStages = 3;
constexpr int kPfSoftmaxWarps = 16;
constexpr int kPfThreads = 64 + 32 * kPfSoftmaxWarps;
constexpr float kPfTau = 8.0f;             // m_w moves once a score passes it by 2^8
constexpr int kPfEMax = 64;                // largest e = m_w - m_O before O is rescaled
constexpr float kPfMaxMove = 16777216.0f;  // cap on one move of m_w, keeps it an exact integer

// Shared memory map (byte offsets from a 1024-aligned base).
struct PfSmem {
    static constexpr int kQ = 0;                                   // 128 rows x 64 B, 64-byte swizzle
    static constexpr int kKBytes = 128 * 64;
    static constexpr int kK = kQ + 128 * 64;                       // per stage: 128 keys x 64 B
    static constexpr int kVRows = 144;                             // 128 channels, ones row, 15 zero rows
    static constexpr int kVBytes = kVRows * 128;
    static constexpr int kVTmaBytes = 128 * 128;
    static constexpr int kV = kK + kPfStages * kKBytes;            // per stage: 144 rows x 128 B, 128-byte swizzle
    static constexpr int kPBuf = 2 * 128 * 128;                    // P_hi then P_lo, 128 rows x 128 B each
    static constexpr int kP = kV + kPfStages * kVBytes;            // 2 buffers
    static constexpr int kSfQ = kP + 2 * kPBuf;                    // 512-byte scale atoms
    static constexpr int kSfK = kSfQ + 512;
    static constexpr int kSfV = kSfK + kPfStages * 512;
    static constexpr int kSfP = kSfV + kPfStages * 512;            // one atom per P buffer (P_hi and P_lo share it)
    static constexpr int kSfOne = kSfP + 2 * 512;
    static constexpr int kXmax = kSfOne + 512;                     // float [4 blocks][128 rows]
    static constexpr int kXe = kXmax + 4 * 128 * 4;                // int [4 blocks][128 rows]
    static constexpr int kVote = kXe + 4 * 128 * 4;                // u32 [4 quarters][2 parities][4 blocks]
    static constexpr int kBar = kVote + 4 * 2 * 4 * 4;
    // kv_full/kv_empty per stage, q_full, patch, s_full x2, p_full x2, pv_done x2,
    // o_final, vote [4 quarters][2], xe [4 quarters].
    static constexpr int kNumBars = 2 * kPfStages + 9 + 8 + 4;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kUsed = kMisc + 16;
    static constexpr int kBytes = kUsed + 1024;  // slack for aligning the base
};
static_assert(PfSmem::kV % 1024 == 0 && PfSmem::kP % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(PfSmem::kBytes <= 227 * 1024, "shared memory budget");

// TMEM columns (512 allocated, one CTA per SM).
constexpr uint32_t kPfTmemCols = 512;
constexpr uint32_t kPfColO = 256;  // 144 columns: O[:, 0:128], the row sum in column 128
constexpr uint32_t kPfColSfQ = 400;
__device__ __forceinline__ uint32_t pf_col_s(int buf) { return 128u * buf; }
__device__ __forceinline__ uint32_t pf_col_sf_k(int buf) { return 404u + 4u * buf; }
// V scales per buffer: 4 columns, then 4 constant columns for the ones row.
__device__ __forceinline__ uint32_t pf_col_sf_v(int buf) { return 412u + 8u * buf; }
__device__ __forceinline__ uint32_t pf_col_sf_p(int buf) { return 428u + 4u * buf; }

constexpr uint32_t pf_idesc(uint32_t fmt, uint32_t n) {
    return (fmt << 7) | (fmt << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}
constexpr uint32_t kPfIdQK = pf_idesc(1u, 128);             // E2M1 x E2M1, N = 128 keys
constexpr uint32_t kPfIdPV = pf_idesc(0u, PfSmem::kVRows);  // E4M3 x E4M3, N = 144
__device__ __forceinline__ uint32_t pf_sf_id(uint32_t idesc, uint32_t id) { return idesc | (id << 29) | (id << 4); }

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

// Wait on an mbarrier phase that every peer reaches within its own bounded
// waits. It does not give up on the abort flag, so all waiters see the same
// phase and take the same branch afterwards.
constexpr uint64_t kPfVoteTimeoutNs = 4 * kWaitTimeoutNs;

__device__ __noinline__ bool pf_wait_peers_slow(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 20000))
        if (globaltimer_ns() - t0 > kPfVoteTimeoutNs) return false;
    return true;
}

__device__ __forceinline__ bool pf_wait_peers(uint64_t *bar, uint32_t parity) {
    return mbar_try_wait(bar, parity) || pf_wait_peers_slow(bar, parity);
}

// O *= 2^-E for the four columns at taddr of this thread's row, E >= 0.
__device__ __noinline__ void pf_rescale_o(uint32_t taddr, int ncols, int E) {
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

struct PfUnit {
    int b, h_q, h_kv, q0, L, T;
};

__device__ __forceinline__ PfUnit pf_unit(const AttnParams &p) {
    PfUnit u;
    const int per = p.B * p.Hq;
    const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / per;  // longest (causal) first
    const int rem = static_cast<int>(blockIdx.x) % per;
    u.b = rem / p.Hq;
    u.h_q = rem % p.Hq;
    u.h_kv = u.h_q / p.G;
    u.q0 = qt * 128;
    const int R = imin(128, p.Sq - u.q0);
    const int L = p.seqlens ? p.seqlens[u.b] : p.Lk;
    u.L = imax(0, imin(L, p.kv_cap));
    int kv_end = u.L;
    if (p.causal) kv_end = imin(u.L, u.q0 + R + u.L - p.Sq);
    u.T = kv_end > 0 ? (kv_end + 127) / 128 : 0;
    return u;
}

}  // namespace

template <bool kStageQK>
__global__ void __launch_bounds__(kPfThreads, 1)
    qk4v8_prefill_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                         const AttnParams p) {
    using S = PfSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const PfUnit u = pf_unit(p);
    const int T = u.T;

    // Softmax thread identity (warps 2..17).
    const int sw = warp - 2;
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int cg = sw >> 2;        // key block within each tile
    const int row = quarter * 32 + lane;
    const int qi = u.q0 + row;
    const bool row_valid = warp >= 2 && qi < p.Sq;

    if (T <= 0 || (p.status && *reinterpret_cast<const volatile int32_t *>(p.status) != 0)) {
        // No key for any row of the tile: O = 0, lse = -inf.
        if (row_valid && !kStageQK) {
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((static_cast<int64_t>(u.b) * p.Sq + qi) * p.Hq + u.h_q) * 128 +
                                                   32 * cg);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(0, 0, 0, 0);
        }
        if (row_valid && cg == 0 && p.lse) p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] = -INFINITY;
        return;
    }

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::kBar);
    uint64_t *kv_full = bars;
    uint64_t *kv_empty = bars + kPfStages;
    uint64_t *q_full = bars + 2 * kPfStages;
    uint64_t *patch = q_full + 1;
    uint64_t *s_full = q_full + 2;   // [2]
    uint64_t *p_full = q_full + 4;   // [2]
    uint64_t *pv_done = q_full + 6;  // [2]
    uint64_t *o_final = q_full + 8;
    uint64_t *vote_bar = q_full + 9;  // [quarter][parity]
    uint64_t *xe_bar = vote_bar + 8;  // [quarter]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMisc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + S::kMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(patch, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], kPfSoftmaxWarps);
            mbar_init(&pv_done[s], 1);
        }
        mbar_init(o_final, 1);
        for (int g = 0; g < 8; ++g) mbar_init(&vote_bar[g], 4);
        for (int g = 0; g < 4; ++g) mbar_init(&xe_bar[g], 4);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kPfTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The last key tile is ragged when L is not a multiple of 128 and in range.
    const bool last_partial = !kStageQK && (u.L & 127) != 0 && T == (u.L + 127) / 128;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            if (!kStageQK) prefetch_tensormap(&tmap_v);
        }
        // Q rows into the 64-byte-swizzled A tile and the Q scale atom; rows past
        // Sq are zero.
        const int64_t qhead = static_cast<int64_t>(u.b) * p.Hq + u.h_q;
        for (int c = lane; c < 512; c += 32) {
            const int r = c >> 2, j = c & 3;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (u.q0 + r < p.Sq)
                val = *reinterpret_cast<const uint4 *>(p.q_codes + (qhead * p.q_cap + u.q0 + r) * 64 + j * 16);
            *reinterpret_cast<uint4 *>(smem + S::kQ + r * 64 + ((j ^ ((r >> 1) & 3)) << 4)) = val;
        }
        {
            // The tile's 128 rows are exactly one 128-token scale block.
            const uint4 *src = reinterpret_cast<const uint4 *>(p.q_scales + (qhead * (p.q_cap / 128) + u.q0 / 128) * 512);
            for (int c = lane; c < 32; c += 32) {
                // 16-byte chunk c holds rows r = c (+32, +64, +96 in its four words)
                uint4 w = src[c];
                if (u.q0 + c >= p.Sq) w.x = 0;
                if (u.q0 + c + 32 >= p.Sq) w.y = 0;
                if (u.q0 + c + 64 >= p.Sq) w.z = 0;
                if (u.q0 + c + 96 >= p.Sq) w.w = 0;
                reinterpret_cast<uint4 *>(smem + S::kSfQ)[c] = w;
            }
        }
        if (!kStageQK) {
            // Constant V rows: row 128 = 1.0 (E4M3 0x38), rows 129..143 = 0, and a
            // scale atom of 2^0 for them.
            for (int s = 0; s < kPfStages; ++s)
                for (int c = lane; c < 16 * 8; c += 32) {
                    const int r = 128 + (c >> 3);
                    const uint32_t fillv = r == 128 ? 0x38383838u : 0u;
                    *reinterpret_cast<uint4 *>(smem + S::kV + s * S::kVBytes + r * 128 + (c & 7) * 16) =
                        make_uint4(fillv, fillv, fillv, fillv);
                }
            reinterpret_cast<uint4 *>(smem + S::kSfOne)[lane] =
                make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && !p.test_stall) mbar_arrive(q_full);

        const int kvh = u.b * p.Hkv + u.h_kv;
        const int nblk = p.kv_cap / 128;
        int issued = 0;
        for (int it = 0; it < T; ++it) {
            const int st = it % kPfStages;
            const uint32_t ph = (it / kPfStages) & 1;
            bool ok = wait_bar(&kv_empty[st], ph ^ 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (lane == 0) {
                const int64_t atom = (static_cast<int64_t>(kvh) * nblk + it) * 512;
                if (kStageQK) {
                    mbar_arrive_expect_tx(&kv_full[st], S::kKBytes + 512);
                } else {
                    mbar_arrive_expect_tx(&kv_full[st], S::kKBytes + S::kVTmaBytes + 1024);
                    tma_load_3d(smem + S::kV + st * S::kVBytes, &tmap_v, it * 128, 0, kvh, &kv_full[st]);
                    bulk_load(smem + S::kSfV + st * 512, p.v_scales + atom, 512, &kv_full[st]);
                }
                tma_load_3d(smem + S::kK + st * S::kKBytes, &tmap_k, 0, it * 128, kvh, &kv_full[st]);
                bulk_load(smem + S::kSfK + st * 512, p.k_scales + atom, 512, &kv_full[st]);
            }
            issued = it + 1;
            if (last_partial && it == T - 1) {
                // Keys at or past L may hold anything (a reused buffer). Their P is
                // zero, but a NaN code or scale in V would still poison O: zero them.
                ok = wait_bar(&kv_full[st], ph, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) break;
                const int jv = u.L - it * 128;  // valid keys in this tile, 1..127
                uint8_t *vt = smem + S::kV + st * S::kVBytes;
                for (int c = lane; c < 128 * 8; c += 32) {
                    const int r = c >> 3, q = c & 7;
                    if (16 * q + 16 <= jv) continue;
                    uint8_t *chunk = vt + r * 128 + ((q ^ (r & 7)) << 4);
                    for (int e = 0; e < 16; ++e)
                        if (16 * q + e >= jv) chunk[e] = 0;
                }
                uint8_t *sfv = smem + S::kSfV + st * 512;
                for (int r = lane; r < 128; r += 32)
                    for (int g = (jv + 31) / 32; g < 4; ++g) sfv[(r & 31) * 16 + (r >> 5) * 4 + g] = 0;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(patch);
            }
        }
        // Let every issued copy land before the CTA can retire.
        if (lane == 0) {
            for (int it = imax(0, issued - kPfStages); it < issued; ++it) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&kv_full[it % kPfStages], (it / kPfStages) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------------- MMA issuer
        // The whole warp runs the loop and waits, so the descriptors stay
        // warp-uniform; one elected lane issues the tcgen05 instructions.
        uint32_t pred;
        asm volatile(
            "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.u32 %0, 1, 0, e;\n\t}"
            : "=r"(pred));
        const bool leader = pred != 0;
        bool ok = __all_sync(0xffffffffu, wait_bar(q_full, 0, abort_flag, p.status));
        if (ok) {
            tc_fence_after();
            const uint32_t sb = smem_u32(smem);
            // Descriptors for stage / buffer 0; the others are fixed offsets of the
            // 14-bit start-address field (16-byte units).
            const uint64_t dQ = smem_desc(sb + S::kQ, 16, 512, 4);
            const uint64_t dK0 = smem_desc(sb + S::kK, 16, 512, 4);
            const uint64_t dV0 = smem_desc(sb + S::kV, 16, 1024, 2);
            const uint64_t dP0 = smem_desc(sb + S::kP, 16, 1024, 2);
            const uint64_t dSfK0 = smem_desc(sb + S::kSfK, 0, 128, 0);
            const uint64_t dSfV0 = smem_desc(sb + S::kSfV, 0, 128, 0);
            const uint64_t dSfP0 = smem_desc(sb + S::kSfP, 0, 128, 0);
            const uint32_t tSfQ = tmem + kPfColSfQ;
            const uint32_t tO = tmem + kPfColO;
            if (leader) {
                tc_cp_32x128b_warpx4(tSfQ, smem_desc(sb + S::kSfQ, 0, 128, 0));
                if (!kStageQK) {
                    const uint64_t dOne = smem_desc(sb + S::kSfOne, 0, 128, 0);
                    tc_cp_32x128b_warpx4(tmem + pf_col_sf_v(0) + 4, dOne);
                    tc_cp_32x128b_warpx4(tmem + pf_col_sf_v(1) + 4, dOne);
                }
            }
            __syncwarp();
            auto issue_pv = [&](int j) -> bool {
                if (!__all_sync(0xffffffffu, wait_bar(&p_full[j & 1], (j >> 1) & 1, abort_flag, p.status)))
                    return false;
                tc_fence_after();
                const int st = j % kPfStages;
                const uint32_t tSfV = tmem + pf_col_sf_v(j & 1);
                const uint32_t tSfP = tmem + pf_col_sf_p(j & 1);
                const uint64_t dV = dV0 + static_cast<uint64_t>(st * (S::kVBytes >> 4));
                const uint64_t dPhi = dP0 + static_cast<uint64_t>((j & 1) * (S::kPBuf >> 4));
                const uint64_t dPlo = dPhi + static_cast<uint64_t>((128 * 128) >> 4);
                if (leader) {
                    tc_cp_32x128b_warpx4(tSfV, dSfV0 + static_cast<uint64_t>(st * 32));
                    tc_cp_32x128b_warpx4(tSfP, dSfP0 + static_cast<uint64_t>((j & 1) * 32));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tO, dPhi + 2 * k, dV + 2 * k, pf_sf_id(kPfIdPV, k), tSfP | (k << 30),
                                    tSfV | (k << 30), (j > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tO, dPlo + 2 * k, dV + 2 * k, pf_sf_id(kPfIdPV, k), tSfP | (k << 30),
                                    tSfV | (k << 30), 1u);
                    tc_commit(&pv_done[j & 1]);
                    tc_commit(&kv_empty[st]);
                }
                __syncwarp();
                return true;
            };
            for (int it = 0; it < T && ok; ++it) {
                const int st = it % kPfStages;
                const int sbuf = it & 1;
                ok = wait_bar(&kv_full[st], (it / kPfStages) & 1, abort_flag, p.status);
                if (ok && last_partial && it == T - 1) ok = wait_bar(patch, 0, abort_flag, p.status);
                // QK-only stage: S buffer `sbuf` is free once the softmax warps have
                // drained tile it-2 (their p_full arrival).
                if (kStageQK && ok && it >= 2) ok = wait_bar(&p_full[sbuf], ((it - 2) >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                const uint32_t tSfK = tmem + pf_col_sf_k(sbuf);
                const uint64_t dK = dK0 + static_cast<uint64_t>(st * (S::kKBytes >> 4));
                const uint32_t tS = tmem + pf_col_s(sbuf);
                if (leader) {
                    tc_cp_32x128b_warpx4(tSfK, dSfK0 + static_cast<uint64_t>(st * 32));
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc_mma_mxf4(tS, dQ + 2 * kk, dK + 2 * kk, pf_sf_id(kPfIdQK, 2 * kk), tSfQ | ((2u * kk) << 30),
                                    tSfK | ((2u * kk) << 30), kk > 0 ? 1u : 0u);
                    tc_commit(&s_full[sbuf]);
                    if (kStageQK) tc_commit(&kv_empty[st]);
                }
                __syncwarp();
                // S buffer (it+1)&1 is reused by QK(it+1) only after p_full of tile
                // it-1, which issue_pv(it-1) waits for here.
                if (!kStageQK && it >= 1) ok = issue_pv(it - 1);
            }
            if (!kStageQK && ok) ok = issue_pv(T - 1);
        }
        // o_final completes once every tcgen05 operation issued above has, also
        // when the loop unwound early, so TMEM is freed with nothing in flight.
        if (leader) tc_commit(o_final);
        __syncwarp();
        (void)pf_wait_peers(o_final, 0);
    } else {
        // ------------------------------------------------------------------ softmax
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int gbar = 1 + quarter;  // named barrier of the row's four threads' warps
        // Exclusive key bound of this row (bottom-right causal alignment).
        int limit = u.L;
        if (p.causal) limit = imin(limit, qi + u.L - p.Sq + 1);
        limit = imax(limit, 0);
        float *xmax = reinterpret_cast<float *>(smem + S::kXmax);
        int *xe = reinterpret_cast<int *>(smem + S::kXe);
        volatile uint32_t *votes = reinterpret_cast<volatile uint32_t *>(smem + S::kVote) + quarter * 8;
        // Byte offset of this thread's two 16-byte chunks in a P tile (128-byte
        // swizzle: chunk c of row r sits at chunk c ^ (r % 8)).
        const int pofs0 = row * 128 + (((2 * cg) ^ (row & 7)) << 4);
        const int pofs1 = row * 128 + (((2 * cg + 1) ^ (row & 7)) << 4);
        const int sf_off = (row & 31) * 16 + (row >> 5) * 4 + cg;
        const float sc = p.scale_log2;
        float mneg = 0.f;  // -m_w (log2 units)
        int e = 0;         // m_w - m_O
        uint32_t n_rescales = 0;
        float qk_rowmax = -INFINITY;  // QK stage: the row's largest scaled score
        bool ok = true;
        for (int it = 0; it < T; ++it) {
            const int sbuf = it & 1;
            ok = __all_sync(0xffffffffu, wait_bar(&s_full[sbuf], (it >> 1) & 1, abort_flag, p.status));
            uint32_t s[32];
            if (ok) {
                tc_fence_after();
                tc_ld_32x32b_x32(tmem + lane_base + pf_col_s(sbuf) + 32 * cg, s);
                tc_wait_ld();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) s[j] = 0xFF800000u;
            }
            if (p.test_dump_s && blockIdx.x == 0 && it == 0) {
#pragma unroll
                for (int j = 0; j < 32; ++j) p.test_dump_s[row * 128 + 32 * cg + j] = __uint_as_float(s[j]);
            }
            // Keys at or past the row's bound are -inf (raw scores; the scale is
            // positive).
            const int jv = imax(0, imin(limit - (it * 128 + 32 * cg), 32));
            if (jv < 32) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j >= jv) s[j] = 0xFF800000u;
            }
            float bm = max32(s) * sc;  // block max, scaled, before subtracting m_w
            if (kStageQK) {
                qk_rowmax = fmaxf(qk_rowmax, bm);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sbuf]);
                if (!ok) break;
                continue;
            }
            if (it == 0) {
                // The row's four threads agree on m_O = m_w: the row's largest score
                // in the first tile. A row with no key there has none at all (its
                // bound does not grow) and keeps m = 0 with a zero sum.
                xmax[cg * 128 + row] = bm;
                bar_sync(gbar, 128);
                const float rm = fmax3(fmaxf(xmax[row], xmax[128 + row]), xmax[256 + row], xmax[384 + row]);
                if (rm > -INFINITY) mneg = -rm;
                bm += mneg;
            } else {
                bm += mneg;
                if (bm > kPfTau) {
                    // Move m_w up to the next whole binade above the block max, so e
                    // stays an integer.
                    const float de = ceilf(fminf(bm, kPfMaxMove));
                    mneg -= de;
                    e += static_cast<int>(de);
                    bm -= de;
                }
            }
            // Vote for the tile: bit 0, some offset of this quarter passed kPfEMax
            // (O must be rescaled before P V of this tile); bit 1, the CTA unwinds.
            const bool over = __any_sync(0xffffffffu, e > kPfEMax);
            if (lane == 0) {
                votes[sbuf * 4 + cg] = (over ? 1u : 0u) | ((!ok || *abort_flag) ? 2u : 0u);
                mbar_arrive(&vote_bar[quarter * 2 + sbuf]);
            }
            // The block's largest p lands in [2^7, 2^8): p' = 2^(s*scale - m_w - x).
            const float xb = fmaxf(floorf(bm) - 7.f, -130.f);
            const float madd = mneg - xb;
            // P_hi = E4M3(p') and P_lo = E4M3(p' - P_hi), through f16 pairs: p' is
            // rounded to f16 (relative error 2^-11, below what P_lo resolves), the
            // value of P_hi comes back exactly as f16, and the difference is exact.
            uint32_t hw[8], lw[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint32_t h01, h23, l01, l23;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int j = 4 * q + 2 * half;
                    const float2 uu = ffma2(make_float2(__uint_as_float(s[j]), __uint_as_float(s[j + 1])),
                                            make_float2(sc, sc), make_float2(madd, madd));
                    const __half2 ph = __floats2half2_rn(exp2_approx(uu.x), exp2_approx(uu.y));
                    const uint32_t phw = *reinterpret_cast<const uint32_t *>(&ph);
                    const uint16_t h2 = cvt_e4m3x2_from_f16x2(phw);
                    const uint32_t hvw = cvt_e4m3x2_to_f16x2(h2);
                    const __half2 d = __hsub2(ph, *reinterpret_cast<const __half2 *>(&hvw));
                    const uint16_t l2 = cvt_e4m3x2_from_f16x2(*reinterpret_cast<const uint32_t *>(&d));
                    if (half == 0) {
                        h01 = h2;
                        l01 = l2;
                    } else {
                        h23 = h2;
                        l23 = l2;
                    }
                }
                hw[q] = h01 | (h23 << 16);
                lw[q] = l01 | (l23 << 16);
            }
            // P buffer `sbuf` was last read by P V of tile it-2.
            if (it >= 2) (void)__all_sync(0xffffffffu, wait_bar(&pv_done[sbuf], ((it >> 1) & 1) ^ 1, abort_flag, p.status));
            // Collect the vote; every warp of the quarter reads the same four words.
            const bool okv = pf_wait_peers(&vote_bar[quarter * 2 + sbuf], (it >> 1) & 1);
            const uint32_t flags =
                okv ? (votes[sbuf * 4] | votes[sbuf * 4 + 1] | votes[sbuf * 4 + 2] | votes[sbuf * 4 + 3]) : 2u;
            if (flags & 2u) {
                ok = false;
                break;
            }
            if (flags & 1u) {
                // Move m_O of each row up by E, the largest offset among the row's four
                // threads (when it passed kPfEMax). O, which holds P V up to tile it-1,
                // is scaled by 2^-E; P bytes are relative to m_w and stay as they are.
                xe[cg * 128 + row] = e;
                __syncwarp();
                if (lane == 0) mbar_arrive(&xe_bar[quarter]);
                const bool okx = pf_wait_peers(&xe_bar[quarter], n_rescales & 1);
                ++n_rescales;
                int E = 0;
                if (okx) {
                    E = imax(imax(xe[row], xe[128 + row]), imax(xe[256 + row], xe[384 + row]));
                    if (E <= kPfEMax) E = 0;
                    e -= E;
                }
                if (okx && it >= 1) {
                    const bool okw = wait_bar(&pv_done[(it - 1) & 1], ((it - 1) >> 1) & 1, abort_flag, p.status);
                    if (__all_sync(0xffffffffu, okw)) {
                        tc_fence_after();
                        // This thread's share of the row's 144 O columns.
                        pf_rescale_o(tmem + lane_base + kPfColO + 36 * cg, 36, E);
                    }
                }
            }
            uint8_t *pb = smem + S::kP + sbuf * S::kPBuf;
            *reinterpret_cast<uint4 *>(pb + pofs0) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4 *>(pb + pofs1) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
            *reinterpret_cast<uint4 *>(pb + 128 * 128 + pofs0) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            *reinterpret_cast<uint4 *>(pb + 128 * 128 + pofs1) = make_uint4(lw[4], lw[5], lw[6], lw[7]);
            // Scale byte of (row, block cg): 2^(e + x), relative to m_O. A block far
            // below m_O clamps at the smallest E8M0 value; it is negligible there.
            smem[S::kSfP + sbuf * 512 + sf_off] =
                static_cast<uint8_t>(imin(254, imax(0, 127 + e + static_cast<int>(xb))));
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[sbuf]);
        }
        // ---------------------------------------------------------------- epilogue
        if (ok) ok = wait_bar(o_final, 0, abort_flag, p.status);
        const bool go = __all_sync(0xffffffffu, ok && !*abort_flag);
        if (kStageQK) {
            xmax[cg * 128 + row] = qk_rowmax;
            bar_sync(gbar, 128);
            if (go && cg == 0 && row_valid && p.lse)
                p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] =
                    fmax3(fmaxf(xmax[row], xmax[128 + row]), xmax[256 + row], xmax[384 + row]);
        } else if (go) {
            tc_fence_after();
            uint32_t o[32];
            tc_ld_32x32b_x32(tmem + lane_base + kPfColO + 32 * cg, o);
            const uint32_t lraw = tc_ld_32x32b_x1(tmem + lane_base + kPfColO + 128);
            tc_wait_ld();
            const float l = __uint_as_float(lraw);
            if (row_valid) {
                // O and l are both relative to m_O = m_w - e.
                const bool any = l > 0.f;
                const float inv = any ? 1.f / l : 0.f;
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((static_cast<int64_t>(u.b) * p.Sq + qi) * p.Hq + u.h_q) * 128 +
                                                       32 * cg);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int c = 8 * q + 2 * k;
                        const __nv_bfloat162 v2 =
                            __floats2bfloat162_rn(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv);
                        w[k] = *reinterpret_cast<const uint32_t *>(&v2);
                    }
                    dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
                }
                if (cg == 0 && p.lse)
                    p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] =
                        any ? (log2f(l) - mneg - static_cast<float>(e)) * 0.6931471805599453f : -INFINITY;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kPfTmemCols);
    }
}

template <bool kStageQK>
static cudaError_t launch_prefill_impl(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, int grid,
                                       cudaStream_t stream) {
    constexpr int kMaxDevices = 64;
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !configured[dev]) {
        e = cudaFuncSetAttribute(qk4v8_prefill_kernel<kStageQK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 PfSmem::kBytes);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) configured[dev] = true;
    }
    qk4v8_prefill_kernel<kStageQK><<<grid, kPfThreads, PfSmem::kBytes, stream>>>(tk, tv, p);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, int grid,
                           cudaStream_t stream) {
    return launch_prefill_impl<false>(tk, tv, p, grid, stream);
}

cudaError_t launch_prefill_stage_qk(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, int grid,
                                    cudaStream_t stream) {
    return launch_prefill_impl<true>(tk, tv, p, grid, stream);
}

}  // namespace qk4v8
