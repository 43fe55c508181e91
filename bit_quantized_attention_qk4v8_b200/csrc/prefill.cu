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
// Softmax: eight warps, two per TMEM lane quarter (query rows 32q .. 32q+31),
// taking alternate key tiles (ping-pong): warp parity pp owns tiles it with
// it % 2 == pp, one query row per thread and all 128 keys of the tile. The
// S accumulator is double-buffered by tile parity, so each warp set has its own
// S buffer, P buffer and barriers, and the tensor core computes S of tile it+2
// while the warps encode P of tile it.
//   - Each warp keeps its own reference max m_w per row: p = 2^(s*scale - m_w)
//     <= 2^8. m_w moves only when a score passes it by 2^8, by whole binades.
//   - The O accumulator has one reference m_O per row, the row max of the
//     first tile. e = m_w - m_O is an integer, carried in the P scale bytes.
//   - Each 32-key block's largest p is brought to about [2^7, 2^8) by a
//     further power of two 2^-x, also in its scale byte: 127 + e + x.
//   - If some e passes 2^64, the tile's owner scales the row of O by 2^-E
//     (after P V of the previous tile, before its own) and lowers e by E.
//     The owner of the next tile learns E (and, after tile 0, m_O) through a
//     one-way handshake posted early in each tile.
// P is kept as two E4M3 terms with the same scales: P_hi = E4M3(p) and
// P_lo = E4M3(p - P_hi), about 8 significant bits. V carries an extra row of
// ones, so O column 128 accumulates the softmax denominator sum(P_hi + P_lo)
// in the same MMAs.
//
// Warp roles (320 threads): warps 0..7 softmax and epilogue, warp 8 TMA
// producer, warp 9 TMEM allocator and MMA issuer.
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

constexpr int kPfKStages = 4;               // K tiles in flight (freed when QK^T of the tile completes)
constexpr int kPfVStages = 4;               // V tiles in flight (freed when P V of the tile completes)
constexpr int kPfSoftmaxWarps = 8;          // two per TMEM lane quarter, alternate key tiles
// Warps 0..7 softmax, then the producer and the MMA issuer.
constexpr int kPfThreads = 32 * kPfSoftmaxWarps + 64;
constexpr int kPfProducerWarp = 8;
constexpr int kPfMmaWarp = 9;
constexpr float kPfTau = 8.0f;              // m_w moves once a score passes it by 2^8
constexpr int kPfEMax = 64;                 // largest e = m_w - m_O before O is rescaled
constexpr float kPfMaxMove = 16777216.0f;   // cap on one move of m_w, keeps it an exact integer

// Shared memory map (byte offsets from a 1024-aligned base).
struct PfSmem {
    static constexpr int kQ = 0;                                   // 128 rows x 64 B, 64-byte swizzle
    static constexpr int kKBytes = 128 * 64;
    static constexpr int kK = kQ + 128 * 64;                       // per stage: 128 keys x 64 B
    static constexpr int kVRows = 144;                             // 128 channels, ones row, 15 zero rows
    static constexpr int kVBytes = kVRows * 128;
    static constexpr int kVTmaBytes = 128 * 128;
    static constexpr int kV = kK + kPfKStages * kKBytes;           // per stage: 144 rows x 128 B, 128-byte swizzle
    static constexpr int kPBuf = 2 * 128 * 128;                    // P_hi then P_lo, 128 rows x 128 B each
    static constexpr int kP = kV + kPfVStages * kVBytes;           // 2 buffers, one per warp parity
    static constexpr int kSfQ = kP + 2 * kPBuf;                    // 512-byte scale atoms
    static constexpr int kSfK = kSfQ + 512;
    static constexpr int kSfV = kSfK + kPfKStages * 512;
    static constexpr int kSfP = kSfV + kPfVStages * 512;           // one atom per P buffer (P_hi and P_lo share it)
    static constexpr int kSfOne = kSfP + 2 * 512;
    // Handshake slots [quarter][tile parity][row (lane)]: the shift E of O, and
    // (tile parity 0 only) the reference m_O.
    static constexpr int kHsE = kSfOne + 512;                      // int [4][2][32]
    static constexpr int kHsM = kHsE + 4 * 2 * 32 * 4;             // float [4][2][32]
    static constexpr int kXmax = kHsM + 4 * 2 * 32 * 4;            // float [2 parities][128 rows] (QK stage)
    static constexpr int kBar = kXmax + 2 * 128 * 4;
    // k_full/k_empty, v_full/v_empty per stage; q_full, patch; s_full, s_free,
    // p_full, pv_done per parity; o_final; handshake [4 quarters][2]; m_O
    // handshake [4 quarters].
    static constexpr int kNumBars = 2 * kPfKStages + 2 * kPfVStages + 2 + 8 + 1 + 8 + 4;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kUsed = kMisc + 16;
    static constexpr int kBytes = kUsed + 1024;  // slack for aligning the base
};
static_assert(PfSmem::kV % 1024 == 0 && PfSmem::kP % 1024 == 0 && PfSmem::kVBytes % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
static_assert(PfSmem::kBar % 8 == 0, "mbarrier alignment");
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

// End of the CTA: every warp arrives here from its own role branch (the
// warpgroups hold different register counts, so they never share this code);
// the MMA warp then frees the tensor memory.
__device__ __forceinline__ void pf_teardown(bool mma_warp, uint32_t tmem, uint32_t ncols) {
    tc_fence_before();
    __syncthreads();
    if (mma_warp) {
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
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

    // Softmax thread identity (warps 0..7): lane quarter, tile parity, query row.
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int pp = warp >> 2;      // the warp owns tiles it with it % 2 == pp
    const int row = quarter * 32 + lane;
    const int qi = u.q0 + row;
    const bool row_valid = warp < kPfSoftmaxWarps && qi < p.Sq;
    // Output channels this warp writes in the epilogue: 64 per parity.
    const int c_lo = 64 * pp;

    if (T <= 0) {
        // No key for any row of the tile: O = 0, lse = -inf.
        if (row_valid && !kStageQK) {
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((static_cast<int64_t>(u.b) * p.Sq + qi) * p.Hq + u.h_q) * 128 +
                                                   c_lo);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_uint4(0, 0, 0, 0);
        }
        if (row_valid && pp == 0 && p.lse) p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] = -INFINITY;
        return;
    }

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::kBar);
    uint64_t *k_full = bars;
    uint64_t *k_empty = k_full + kPfKStages;
    uint64_t *v_full = k_empty + kPfKStages;
    uint64_t *v_empty = v_full + kPfVStages;
    uint64_t *q_full = v_empty + kPfVStages;
    uint64_t *patch = q_full + 1;
    uint64_t *s_full = patch + 1;    // [parity]
    uint64_t *s_free = s_full + 2;   // [parity]
    uint64_t *p_full = s_free + 2;   // [parity]
    uint64_t *pv_done = p_full + 2;  // [parity]
    uint64_t *o_final = pv_done + 2;
    uint64_t *hs_bar = o_final + 1;  // [quarter][parity]
    uint64_t *mo_bar = hs_bar + 8;   // [quarter]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMisc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + S::kMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPfKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kPfVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(patch, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], 4);
            mbar_init(&p_full[s], 4);
            mbar_init(&pv_done[s], 1);
        }
        mbar_init(o_final, 1);
        for (int g = 0; g < 8; ++g) mbar_init(&hs_bar[g], 1);
        for (int g = 0; g < 4; ++g) mbar_init(&mo_bar[g], 1);
        // A status already set by another launch or CTA: unwind at once (every
        // wait returns false), uniformly for the whole CTA.
        *abort_flag = (p.status && *reinterpret_cast<const volatile int32_t *>(p.status) != 0) ? 1u : 0u;
        fence_barrier_init();
    }
    if (warp == kPfMmaWarp) {
        tmem_alloc(tmem_slot, kPfTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The last key tile is ragged when L is not a multiple of 128 and in range.
    const bool last_partial = !kStageQK && (u.L & 127) != 0 && T == (u.L + 127) / 128;

    if (warp == kPfProducerWarp) {
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
            // The tile's 128 rows are exactly one 128-token scale block; 16-byte
            // chunk c holds rows c, c+32, c+64, c+96 in its four words.
            const uint4 *src = reinterpret_cast<const uint4 *>(p.q_scales + (qhead * (p.q_cap / 128) + u.q0 / 128) * 512);
            uint4 w = src[lane];
            if (u.q0 + lane >= p.Sq) w.x = 0;
            if (u.q0 + lane + 32 >= p.Sq) w.y = 0;
            if (u.q0 + lane + 64 >= p.Sq) w.z = 0;
            if (u.q0 + lane + 96 >= p.Sq) w.w = 0;
            reinterpret_cast<uint4 *>(smem + S::kSfQ)[lane] = w;
        }
        if (!kStageQK) {
            // Constant V rows: row 128 = 1.0 (E4M3 0x38), rows 129..143 = 0, and a
            // scale atom of 2^0 for them.
            for (int s = 0; s < kPfVStages; ++s)
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
        // K runs one tile ahead of V: the K ring frees as soon as QK^T of a tile
        // completes, the V ring only after its P V.
        int k_issued = 0, v_issued = 0;
        bool ok = true;
        for (int it = 0; it <= T && ok; ++it) {
            if (it < T) {
                const int st = it % kPfKStages;
                ok = __all_sync(0xffffffffu, wait_bar(&k_empty[st], ((it / kPfKStages) & 1) ^ 1, abort_flag, p.status));
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&k_full[st], S::kKBytes + 512);
                    tma_load_3d(smem + S::kK + st * S::kKBytes, &tmap_k, 0, it * 128, kvh, &k_full[st]);
                    bulk_load(smem + S::kSfK + st * 512, p.k_scales + (static_cast<int64_t>(kvh) * nblk + it) * 512, 512,
                              &k_full[st]);
                }
                k_issued = it + 1;
            }
            const int jt = it - 1;  // V tile issued in this round
            if (kStageQK || jt < 0) continue;
            const int sv = jt % kPfVStages;
            const uint32_t ph = (jt / kPfVStages) & 1;
            ok = __all_sync(0xffffffffu, wait_bar(&v_empty[sv], ph ^ 1, abort_flag, p.status));
            if (!ok) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&v_full[sv], S::kVTmaBytes + 512);
                tma_load_3d(smem + S::kV + sv * S::kVBytes, &tmap_v, jt * 128, 0, kvh, &v_full[sv]);
                bulk_load(smem + S::kSfV + sv * 512, p.v_scales + (static_cast<int64_t>(kvh) * nblk + jt) * 512, 512,
                          &v_full[sv]);
            }
            v_issued = jt + 1;
            if (last_partial && jt == T - 1) {
                // Keys at or past L may hold anything (a reused buffer). Their P is
                // zero, but a NaN code or scale in V would still poison O: zero them.
                ok = __all_sync(0xffffffffu, wait_bar(&v_full[sv], ph, abort_flag, p.status));
                if (!ok) break;
                const int jv = u.L - jt * 128;  // valid keys in this tile, 1..127
                uint8_t *vt = smem + S::kV + sv * S::kVBytes;
                for (int c = lane; c < 128 * 8; c += 32) {
                    const int r = c >> 3, q = c & 7;
                    if (16 * q + 16 <= jv) continue;
                    uint8_t *chunk = vt + r * 128 + ((q ^ (r & 7)) << 4);
                    for (int e = 0; e < 16; ++e)
                        if (16 * q + e >= jv) chunk[e] = 0;
                }
                uint8_t *sfv = smem + S::kSfV + sv * 512;
                for (int r = lane; r < 128; r += 32)
                    for (int g = (jv + 31) / 32; g < 4; ++g) sfv[(r & 31) * 16 + (r >> 5) * 4 + g] = 0;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(patch);
            }
        }
        // Let every issued copy land before the CTA can retire.
        if (lane == 0) {
            for (int it = imax(0, k_issued - kPfKStages); it < k_issued; ++it) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&k_full[it % kPfKStages], (it / kPfKStages) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
            for (int it = imax(0, v_issued - kPfVStages); it < v_issued; ++it) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&v_full[it % kPfVStages], (it / kPfVStages) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
        }
    } else if (warp == kPfMmaWarp) {
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
            // S(i) = Q K(i)^T into S buffer i & 1, once K(i) has landed and the warps
            // of parity i & 1 have read S(i-2) out of that buffer.
            auto issue_qk = [&](int i) -> bool {
                const int st = i % kPfKStages;
                bool w = wait_bar(&k_full[st], (i / kPfKStages) & 1, abort_flag, p.status);
                if (w && i >= 2) w = wait_bar(&s_free[i & 1], ((i - 2) >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, w)) return false;
                tc_fence_after();
                const uint32_t tSfK = tmem + pf_col_sf_k(i & 1);
                const uint64_t dK = dK0 + static_cast<uint64_t>(st * (S::kKBytes >> 4));
                const uint32_t tS = tmem + pf_col_s(i & 1);
                if (leader) {
                    tc_cp_32x128b_warpx4(tSfK, dSfK0 + static_cast<uint64_t>(st * 32));
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc_mma_mxf4(tS, dQ + 2 * kk, dK + 2 * kk, pf_sf_id(kPfIdQK, 2 * kk), tSfQ | ((2u * kk) << 30),
                                    tSfK | ((2u * kk) << 30), kk > 0 ? 1u : 0u);
                    tc_commit(&s_full[i & 1]);
                    tc_commit(&k_empty[st]);
                }
                __syncwarp();
                return true;
            };
            // O += P(i) V(i), once V(i) has landed and the warps of parity i & 1
            // have written P(i).
            auto issue_pv = [&](int i) -> bool {
                const int sv = i % kPfVStages;
                bool w = wait_bar(&v_full[sv], (i / kPfVStages) & 1, abort_flag, p.status);
                if (w && last_partial && i == T - 1) w = wait_bar(patch, 0, abort_flag, p.status);
                if (w) w = wait_bar(&p_full[i & 1], (i >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, w)) return false;
                tc_fence_after();
                const uint32_t tSfV = tmem + pf_col_sf_v(i & 1);
                const uint32_t tSfP = tmem + pf_col_sf_p(i & 1);
                const uint64_t dV = dV0 + static_cast<uint64_t>(sv * (S::kVBytes >> 4));
                const uint64_t dPhi = dP0 + static_cast<uint64_t>((i & 1) * (S::kPBuf >> 4));
                const uint64_t dPlo = dPhi + static_cast<uint64_t>((128 * 128) >> 4);
                if (leader) {
                    tc_cp_32x128b_warpx4(tSfV, dSfV0 + static_cast<uint64_t>(sv * 32));
                    tc_cp_32x128b_warpx4(tSfP, dSfP0 + static_cast<uint64_t>((i & 1) * 32));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tO, dPhi + 2 * k, dV + 2 * k, pf_sf_id(kPfIdPV, k), tSfP | (k << 30),
                                    tSfV | (k << 30), (i > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tO, dPlo + 2 * k, dV + 2 * k, pf_sf_id(kPfIdPV, k), tSfP | (k << 30),
                                    tSfV | (k << 30), 1u);
                    tc_commit(&pv_done[i & 1]);
                    tc_commit(&v_empty[sv]);
                }
                __syncwarp();
                return true;
            };
            // Order: S(0), S(1), then per tile i: S(i+2) as soon as S(i) has been
            // read (early in tile i's softmax), then P(i) V(i) once P(i) is written.
            ok = issue_qk(0);
            if (ok && T > 1) ok = issue_qk(1);
            for (int i = 0; i < T && ok; ++i) {
                if (i + 2 < T) ok = issue_qk(i + 2);
                if (ok && !kStageQK) ok = issue_pv(i);
            }
        }
        // o_final completes once every tcgen05 operation issued above has, also
        // when the loop unwound early, so TMEM is freed with nothing in flight.
        if (leader) tc_commit(o_final);
        __syncwarp();
        (void)pf_wait_peers(o_final, 0);
    } else {
        // ------------------------------------------------------------------ softmax
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        // Exclusive key bound of this row (bottom-right causal alignment).
        int limit = u.L;
        if (p.causal) limit = imin(limit, qi + u.L - p.Sq + 1);
        limit = imax(limit, 0);
        // Handshake slots of this thread's row (shared-space addresses), E and m
        // by tile parity.
        const uint32_t a_e = smem_u32(smem + S::kHsE) + quarter * 256 + lane * 4;
        const uint32_t a_m = smem_u32(smem + S::kHsM) + quarter * 256 + lane * 4;
        uint64_t *hs = hs_bar + quarter * 2;
        uint8_t *pbuf = smem + S::kP + pp * S::kPBuf;
        const int swz = row & 7;
        const float sc = p.scale_log2;
        float mneg = 0.f;  // -m_w (log2 units)
        int e = 0;         // m_w - m_O
        float qk_rowmax = -INFINITY;
        bool ok = true;

        // Handshakes from the other warp of this quarter. The m_O handshake (once,
        // early in tile 0) gives the reference of O; the handshake of tile j (at its
        // end) gives the shift E applied to O before P V(j).
        auto receive_mo = [&]() -> bool {
            if (!__all_sync(0xffffffffu, wait_bar(&mo_bar[quarter], 0, abort_flag, p.status))) return false;
            const float m0 = __uint_as_float(lds32(a_m));
            mneg = m0 > -INFINITY ? -m0 : 0.f;
            e = 0;
            return true;
        };
        auto receive = [&](int j) -> bool {
            if (!__all_sync(0xffffffffu, wait_bar(&hs[j & 1], (j >> 1) & 1, abort_flag, p.status))) return false;
            e -= static_cast<int>(lds32(a_e + (j & 1) * 128));
            return true;
        };

        for (int i = pp; i < T; i += 2) {
            const int k = i >> 1;  // this warp's tile count: phase parity of its barriers
            ok = __all_sync(0xffffffffu, wait_bar(&s_full[pp], k & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            const int jv = imax(0, imin(limit - i * 128, 128));  // keys j < jv are allowed
            int eb[4];  // e + x of each block when it was encoded
            // The tile in two halves of 64 keys, to bound the registers held at once.
            // S is released to the tensor core once the second half has been read.
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t sh[64];
                uint32_t pw[32];  // this half's P bytes: P_hi words [0, 16), P_lo words [16, 32)
                tc_ld_32x32b_x32(tmem + lane_base + pf_col_s(pp) + 64 * hh,
                                 *reinterpret_cast<uint32_t (*)[32]>(&sh[0]));
                tc_ld_32x32b_x32(tmem + lane_base + pf_col_s(pp) + 64 * hh + 32,
                                 *reinterpret_cast<uint32_t (*)[32]>(&sh[32]));
                tc_wait_ld();
                if (hh == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s_free[pp]);  // the tensor core may now compute S(i+2)
                }
                if (p.test_dump_s && blockIdx.x == 0 && i == 0) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) p.test_dump_s[row * 128 + 64 * hh + j] = __uint_as_float(sh[j]);
                }
                // Keys at or past the row's bound are -inf (raw scores; the scale is positive).
                if (jv < 64 * hh + 64) {
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (64 * hh + j >= jv) sh[j] = 0xFF800000u;
                }
                const float bmx0 = max32(*reinterpret_cast<const uint32_t (*)[32]>(&sh[0])) * sc;
                const float bmx1 = max32(*reinterpret_cast<const uint32_t (*)[32]>(&sh[32])) * sc;
                const float hm = fmaxf(bmx0, bmx1);
                if (kStageQK) {
                    qk_rowmax = fmaxf(qk_rowmax, hm);
                    continue;
                }
                if (i == 0 && hh == 0) {
                    // The first half of tile 0 fixes m_O = m_w: the row's largest score
                    // there. It holds key 0, so a row with no key in it has none at all.
                    // Its handshake, posted now, gives m_O to the owner of tile 1.
                    mneg = hm > -INFINITY ? -hm : 0.f;
                    e = 0;
                    sts32(a_m, __float_as_uint(-mneg));
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&mo_bar[quarter]);
                } else if (i == 1 && hh == 0 && !receive_mo()) {
                    ok = false;
                    break;
                }
                {
                    // m_w moves to the next whole binade above the half's max, so e
                    // stays integral.
                    const float bt = hm + mneg;
                    if (bt > kPfTau) {
                        const float de = ceilf(fminf(bt, kPfMaxMove));
                        mneg -= de;
                        e += static_cast<int>(de);
                    }
                }
#pragma unroll
                for (int b2 = 0; b2 < 2; ++b2) {
                    const int b = 2 * hh + b2;
                    // P = 2^(s*scale - m_w - x), x bringing the block max to about
                    // [2^7, 2^8): x = round(bm - 1/2) - 7, without a float-to-int
                    // conversion (the sum with 1.5 * 2^23 rounds to an integer held
                    // in the low mantissa bits).
                    const float bm = fmaxf((b2 ? bmx1 : bmx0) + mneg, -200.f);
                    const float t = (bm - 0.5f) + 12582912.0f;
                    eb[b] = e + (__float_as_int(t) - 0x4B400000) - 7;
                    const float madd = mneg - ((t - 12582912.0f) - 7.0f);
                    // P_hi = E4M3(p), P_lo = E4M3(p - P_hi) through f16 pairs: p is
                    // rounded to f16 (relative error 2^-11, below what P_lo resolves),
                    // the value of P_hi comes back exactly as f16 and the difference
                    // is exact.
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint32_t hh2[2], ll2[2];
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const int j = 32 * b2 + 4 * q + 2 * half;
                            const float y0 = exp2_approx(fmaf(__uint_as_float(sh[j]), sc, madd));
                            const float y1 = exp2_approx(fmaf(__uint_as_float(sh[j + 1]), sc, madd));
                            const __half2 ph = __floats2half2_rn(y0, y1);
                            const uint32_t phw = *reinterpret_cast<const uint32_t *>(&ph);
                            const uint16_t h2 = cvt_e4m3x2_from_f16x2(phw);
                            const uint32_t hvw = cvt_e4m3x2_to_f16x2(h2);
                            const __half2 d = __hsub2(ph, *reinterpret_cast<const __half2 *>(&hvw));
                            hh2[half] = h2;
                            ll2[half] = cvt_e4m3x2_from_f16x2(*reinterpret_cast<const uint32_t *>(&d));
                        }
                        pw[8 * b2 + q] = __byte_perm(hh2[0], hh2[1], 0x5410);
                        pw[16 + 8 * b2 + q] = __byte_perm(ll2[0], ll2[1], 0x5410);
                    }
                }
                // P buffer pp was last read by P V(i-2), issued at the end of this
                // warp's previous tile.
                if (hh == 0 && i >= 2 &&
                    !__all_sync(0xffffffffu, wait_bar(&pv_done[pp], (k - 1) & 1, abort_flag, p.status))) {
                    ok = false;
                    break;
                }
                const uint32_t prow = smem_u32(pbuf) + row * 128;
#pragma unroll
                for (int c2 = 0; c2 < 4; ++c2) {
                    const uint32_t cofs = static_cast<uint32_t>(((4 * hh + c2) ^ swz) << 4);
                    sts128(prow + cofs, pw[4 * c2], pw[4 * c2 + 1], pw[4 * c2 + 2], pw[4 * c2 + 3]);
                    sts128(prow + 128 * 128 + cofs, pw[16 + 4 * c2], pw[17 + 4 * c2], pw[18 + 4 * c2], pw[19 + 4 * c2]);
                }
            }
            if (!ok) break;
            if (kStageQK) continue;
            // Handshake with the other warp of this quarter, at the end of the tile:
            // take the shift E of tile i-1 (it moved m_O), then decide this tile's.
            const int e_enc = e;
            if (i >= 1 && !receive(i - 1)) {
                ok = false;
                break;
            }
            int E = 0;
            if (e > kPfEMax) {
                E = e;
                e = 0;
            }
            const bool any = __any_sync(0xffffffffu, E != 0);
            if (any && i >= 1) {
                // O holds P V up to tile i-1 (the other warp's): wait for it, then
                // scale this quarter's rows by 2^-E before P V(i).
                if (!__all_sync(0xffffffffu,
                                wait_bar(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, p.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                pf_rescale_o(tmem + lane_base + kPfColO, 144, E);
            }
            // A warp that unwinds posts nothing; its peer's bounded wait then sees
            // the abort flag.
            sts32(a_e + (i & 1) * 128, static_cast<uint32_t>(E));
            __syncwarp();
            if (lane == 0) mbar_arrive(&hs[i & 1]);
            // Scale bytes of (row, block b): 2^(e + x) relative to m_O, with the
            // block's own e and the shifts of m_O since it was encoded. A block far
            // below m_O clamps at the smallest E8M0 value; it is negligible there.
            const int de_o = e - e_enc;
            uint32_t sfw = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) sfw |= static_cast<uint32_t>(imin(254, imax(0, 127 + eb[b] + de_o))) << (8 * b);
            sts32(smem_u32(smem + S::kSfP + pp * 512 + (row & 31) * 16 + (row >> 5) * 4), sfw);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[pp]);
        }
        // The warp that does not own the last tile still applies its handshake, so
        // both warps of the quarter end with the same m_O = m_w - e.
        if (!kStageQK && ok && ((T - 1) & 1) != pp) {
            if (T == 1) ok = receive_mo();  // this warp had no tile: take m_O first
            if (ok) ok = receive(T - 1);
        }

        // ---------------------------------------------------------------- epilogue
        if (ok) ok = wait_bar(o_final, 0, abort_flag, p.status);
        const bool go = __all_sync(0xffffffffu, ok && !*abort_flag);
        if (kStageQK) {
            float *xmax = reinterpret_cast<float *>(smem + S::kXmax);
            xmax[pp * 128 + row] = qk_rowmax;
            bar_sync(1 + quarter, 64);
            if (go && pp == 0 && row_valid && p.lse)
                p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] = fmaxf(xmax[row], xmax[128 + row]);
        } else if (go) {
            tc_fence_after();
            const float l = __uint_as_float(tc_ld_32x32b_x1(tmem + lane_base + kPfColO + 128));
            tc_wait_ld();
            // O and l are both relative to m_O = m_w - e.
            const bool any = l > 0.f;
            // Approximate reciprocal and log2 (no slow-path subroutine, which a
            // register-split region cannot call); both far inside bf16 / lse precision.
            const float inv = any ? __fdividef(1.f, l) : 0.f;
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((static_cast<int64_t>(u.b) * p.Sq + qi) * p.Hq + u.h_q) * 128 +
                                                   c_lo);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t o[32];
                tc_ld_32x32b_x32(tmem + lane_base + kPfColO + c_lo + 32 * h, o);
                tc_wait_ld();
                if (row_valid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const int c = 8 * q + 2 * kk;
                            const __nv_bfloat162 v2 =
                                __floats2bfloat162_rn(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv);
                            w[kk] = *reinterpret_cast<const uint32_t *>(&v2);
                        }
                        dst[4 * h + q] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            if (row_valid && pp == 0 && p.lse)
                p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] =
                    any ? (__log2f(l) - mneg - static_cast<float>(e)) * 0.6931471805599453f : -INFINITY;
        }
    }
    pf_teardown(warp == kPfMmaWarp, tmem, kPfTmemCols);
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
