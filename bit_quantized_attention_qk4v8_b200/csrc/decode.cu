// Split-KV decode / speculative-verify kernel for QK4V8 attention on sm_100a.
//
// Decode is bound by streaming the packed KV cache (MpFA QK4V8 article,
// section 1.3: decode attention is memory bound, and narrower QK cuts the
// traffic). Each CTA streams one contiguous split of one (sequence, KV head)
// cache at HBM rate with TMA.
//
// Orientation ("swap AB"): the 128-token key tile is the MMA's M side, and the
// G*nq query rows of the GQA group (padded to NT = 16, 32 or 64) are its N side:
//   S^T[token][row] = K_tile . Q^T              tcgen05 kind::mxf4 (K, Q scales in TMEM)
//   O^T[chan][row]  += V^T . [P_hi ; P_lo]^T     tcgen05 kind::mxf8f6f4, N = 2*NT
// P_hi and P_lo are stacked along N with per-row E8M0 scales 2^0 and 2^-5, so
// one set of four MMAs per tile accumulates both terms: O^T columns [0, NT)
// hold the P_hi part and [NT, 2NT) the P_lo part, summed in the epilogue.
//
// Softmax: thread (lane quarter q, lane l) owns token 32q + l of the tile; a
// warp covers NC query rows, and the four warps of a column group cover the
// tile's four 32-key blocks. The P operand carries one E8M0 scale per (row,
// 32-key block), so every warp keeps its own reference max m per row: p =
// 2^(s - m) <= 2^8, and the block's scale byte holds the integer offset e =
// m - m_O from the reference m_O of the O accumulator. A warp moves its m (by
// whole binades, only when a score passes it by 2^8) without talking to the
// other warps; the group agrees on m_O once, on its first tile, and moves it
// only when some offset passes 2^64 (an mbarrier vote posted early in the tile
// and collected after the encode, so it rarely waits).
// P_hi = E4M3(p), P_lo = E4M3((p - P_hi) * 32): about 8 significant bits.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer,
// warps 2.. softmax and epilogue (4 per column group of NC rows).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mx_encode.cuh"
#include "pipeline.cuh"
#include "ptx.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

namespace {

constexpr float kTauD = 8.0f;      // a warp moves m once a score passes it by 2^kTauD
constexpr int kEMaxD = 64;         // largest offset e = m - m_O before O itself is rescaled
constexpr float kMaxMoveD = 16777216.0f;  // cap on one move of m (binades), keeps it an exact integer
// Stages of the G*nq <= 16 instantiation, small enough for two CTAs per SM.
// K/V stages of the instances for up to 8 and up to 16 query rows per KV head:
// two CTAs per SM share its 228 KB (each CTA's dynamic shared memory plus the
// 1 KB the hardware keeps per CTA), which leaves room for four stages up to 8
// rows and three for 16.
constexpr int kDecodeStages8 = 4, kDecodeStages16 = 3;
constexpr int kSmemPerSm = 228 * 1024, kSmemReservedPerCta = 1024;
constexpr uint32_t kPhiScaleWord = 0x7F7F7F7Fu;  // E8M0 2^0 for P_hi rows
constexpr uint32_t kPloScaleWord = 0x7A7A7A7Au;  // E8M0 2^-5 for P_lo rows
// Named barriers: one per column group (ids 1..4), and one over all softmax warps.
constexpr int kBarGroup0 = 1, kBarAllSoftmax = 5;
// Limit on the vote wait, which ignores the abort flag so that a column group
// always takes the same branch (nanoseconds; above any bounded wait a peer may
// be sitting in).
constexpr uint64_t kVoteTimeoutNs = 4 * kWaitTimeoutNs;

// NT: query rows of the MMA (its N, at least 16); RW: rows the softmax warps
// cover (RW <= NT, the launch's G*nq at most); NC: rows per softmax warp.
template <int NT, int RW, int NC, int ST>
struct DecodeLayout {
    static_assert(RW <= NT && RW % NC == 0 && NC % 4 == 0, "row split");
    static_assert(RW == NC || NC % 8 == 0, "column groups start at multiples of 8 rows (P^T swizzle)");
    static constexpr int kStages = ST;             // K/V pipeline stages
    static constexpr int kCG = RW / NC;            // column groups
    static constexpr int kSoftmaxWarps = 4 * kCG;
    static constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
    static constexpr int kThreads = 64 + kSoftmaxThreads;
    static constexpr int kQ = 0;  // NT rows x 64 B, 64-byte swizzle
    static constexpr int kK = NT * 64 < 1024 ? 1024 : NT * 64;
    static constexpr int kKBytes = 128 * 64;
    static constexpr int kV = kK + ST * kKBytes;
    static constexpr int kVBytes = 128 * 128;
    static constexpr int kP = kV + ST * kVBytes;  // 2 buffers of [P_hi rows; P_lo rows] x 128 B
    static constexpr int kPBytes = 2 * NT * 128;
    static constexpr int kSfQ = kP + 2 * kPBytes;
    static constexpr int kSfK = kSfQ + 512;
    static constexpr int kSfV = kSfK + ST * 512;
    static constexpr int kSfP = kSfV + ST * 512;  // one P scale atom per P buffer
    // Exchange buffers, each [column group][quarter][NC] 32-bit words, and the
    // row references [softmax warp][NC]: kSoftmaxWarps * NC words, in 128-byte
    // units (the small instances fit four K/V stages beside a second CTA).
    static constexpr int kRowBytes = (kSoftmaxWarps * NC * 4 + 127) / 128 * 128;
    static constexpr int kXmax = kSfP + 1024;       // first-tile row maxima
    static constexpr int kXe = kXmax + kRowBytes;   // offsets e, when O is rescaled
    static constexpr int kLsum = kXe + kRowBytes;   // epilogue row sums
    static constexpr int kEsum = kLsum + kRowBytes;  // epilogue offsets e
    static constexpr int kLim = kEsum + kRowBytes;  // [NT] int: exclusive key bound per query row
    static constexpr int kVote = kLim + (NT * 4 < 128 ? 128 : NT * 4);  // [column group][tile parity][quarter] u32 votes
    static constexpr int kMneg = kVote + 128;       // [softmax warp][NC] float: -m of each row
    static constexpr int kBar = kMneg + kRowBytes;
    // kv_full/empty per stage, q_full, patch, s_full x2, p_full x2, pv_done x2,
    // s_free x2,
    // o_final, vote x2 and e exchange per column group.
    static constexpr int kNumBars = 2 * ST + 9 + 3 * kCG + 2;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16 + 1024;
    // TMEM columns: S^T x2 [0, 2NT), O^T [2NT, 4NT), then scale factors:
    // Q at 4NT, K x2 at 4NT+4, V x2 at 4NT+12, P x2 at 4NT+20.
    static constexpr uint32_t kColO = 2 * NT;
    static constexpr uint32_t kColSfQ = 4 * NT;
    static constexpr uint32_t kTmemCols = 4 * NT + 28 <= 128 ? 128 : (4 * NT + 28 <= 256 ? 256 : 512);
    static_assert(kCG * 4 * NC * 4 <= kRowBytes, "exchange buffers");
    static_assert(kSoftmaxWarps * NC * 4 <= kRowBytes && kMneg % 16 == 0, "row references");
    static_assert(NC <= 32 && NT <= 64, "one lane per row of a warp");
    static_assert(kBytes <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint32_t col_sf_k_d(int nt, int buf) { return static_cast<uint32_t>(4 * nt + 4 + 4 * buf); }
__device__ __forceinline__ uint32_t col_sf_v_d(int nt, int buf) { return static_cast<uint32_t>(4 * nt + 12 + 4 * buf); }
__device__ __forceinline__ uint32_t col_sf_p_d(int nt, int buf) { return static_cast<uint32_t>(4 * nt + 20 + 4 * buf); }

constexpr uint32_t idesc_d(uint32_t fmt, uint32_t n) {
    return (fmt << 7) | (fmt << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}
__device__ __forceinline__ uint32_t sf_id_d(uint32_t idesc, uint32_t id) { return idesc | (id << 29) | (id << 4); }

// tcgen05.ld / st of NC consecutive 32-bit columns for this warp's 32 lanes.
template <int NC>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t (&r)[NC]) {
    static_assert(NC % 4 == 0, "column count");
#pragma unroll
    for (int c = 0; c < NC; c += 4) {
        uint32_t *d = &r[c];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                     : "r"(taddr + c));
    }
}

template <int NC>
__device__ __forceinline__ void tmem_store_cols(uint32_t taddr, const uint32_t (&r)[NC]) {
    static_assert(NC % 4 == 0, "column count");
#pragma unroll
    for (int c = 0; c < NC; c += 4) {
        const uint32_t *d = &r[c];
        asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr + c), "r"(d[0]),
                     "r"(d[1]), "r"(d[2]), "r"(d[3])
                     : "memory");
    }
}

// Low byte of v to shared address addr + kOff (the offset folds into the store).
template <int kOff>
__device__ __forceinline__ void sts_u8(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b8 [%0+%2], %1;" ::"r"(addr), "r"(v), "n"(kOff) : "memory");
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// Stores the P^T bytes of query rows i and i+1 (P_hi rows at 0, P_lo rows at
// NT*128) for this thread's token. pa is the token's byte in row 0; the
// 128-byte swizzle moves row r's byte to 16-byte chunk (chunk ^ (r % 8)), so row
// r sits at (pa ^ ((r & 7) << 4)) + r * 128 (the buffer base is 1024-aligned).
template <int NT, int I>
__device__ __forceinline__ void store_p_pair(uint32_t pa, uint32_t h2, uint32_t l2) {
    const uint32_t a0 = pa ^ static_cast<uint32_t>((I & 7) << 4);
    const uint32_t a1 = pa ^ static_cast<uint32_t>(((I + 1) & 7) << 4);
    sts_u8<I * 128>(a0, h2);
    sts_u8<I * 128 + NT * 128>(a0, l2);
    sts_u8<(I + 1) * 128>(a1, h2 >> 8);
    sts_u8<(I + 1) * 128 + NT * 128>(a1, l2 >> 8);
}

template <int NT, int I, int NC>
struct StorePairs {
    __device__ __forceinline__ static void run(uint32_t pa, const uint32_t (&h)[NC / 2], const uint32_t (&l)[NC / 2]) {
        store_p_pair<NT, I>(pa, h[I / 2], l[I / 2]);
        StorePairs<NT, I + 2, NC>::run(pa, h, l);
    }
};
template <int NT, int NC>
struct StorePairs<NT, NC, NC> {
    __device__ __forceinline__ static void run(uint32_t, const uint32_t (&)[NC / 2], const uint32_t (&)[NC / 2]) {}
};

// Wait on an mbarrier phase that every peer reaches within its own bounded
// waits. Unlike wait_bar it does not give up on the abort flag, so all waiters
// see the same phase and take the same branch afterwards.
__device__ __noinline__ bool wait_bar_peers_slow(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 20000))
        if (globaltimer_ns() - t0 > kVoteTimeoutNs) return false;
    return true;
}

__device__ __forceinline__ bool wait_bar_peers(uint64_t *bar, uint32_t parity) {
    return mbar_try_wait(bar, parity) || wait_bar_peers_slow(bar, parity);
}

// One lane of the (fully active) warp, chosen by elect.sync.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// 2^-k as a float for an integer k >= 0 (0 once it would be subnormal).
__device__ __forceinline__ float exp2_neg_int(int k) {
    return k < 126 ? __uint_as_float(static_cast<uint32_t>(127 - k) << 23) : 0.f;
}

// O *= 2^-E_c for the nc columns at taddr (P_hi part) and taddr + nt (P_lo
// part), E_c held by lane c of the warp. Kept out of line: it runs only when a
// row's reference moves past kEMaxD.
__device__ __noinline__ void rescale_o_cols(uint32_t taddr, int nt, int nc, int E) {
    for (int c8 = 0; c8 < nc; c8 += 8) {
        uint32_t ohi[8], olo[8];
        tmem_load_cols<8>(taddr + c8, ohi);
        tmem_load_cols<8>(taddr + nt + c8, olo);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float a = exp2_neg_int(__shfl_sync(0xffffffffu, E, c8 + c));
            ohi[c] = __float_as_uint(__uint_as_float(ohi[c]) * a);
            olo[c] = __float_as_uint(__uint_as_float(olo[c]) * a);
        }
        tmem_store_cols<8>(taddr + c8, ohi);
        tmem_store_cols<8>(taddr + nt + c8, olo);
    }
    tc_wait_st();
}

}  // namespace

// kExt: the instance for draft-block windows, paged caches and MXFP4 V (the
// QK4V4 comparison point); the other is the plain decode over a contiguous
// MXFP8-V cache.
template <int NT, int RW, int NC, int ST, int MINB, bool kExt>
__global__ void __launch_bounds__(DecodeLayout<NT, RW, NC, ST>::kThreads, MINB)
    qk4v8_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                        const AttnParams p) {
    using Lay = DecodeLayout<NT, RW, NC, ST>;
    constexpr int kStagesD = Lay::kStages;
    constexpr int kSoftmaxThreads = Lay::kSoftmaxThreads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int split = static_cast<int>(blockIdx.x) % p.num_splits;
    const int rem = static_cast<int>(blockIdx.x) / p.num_splits;
    const int h_kv = rem % p.Hkv;
    const int b = rem / p.Hkv;
    const int nq = p.Sq;
    const int R = p.G * nq;
    const int L = imax(0, imin(p.seqlens[b], p.kv_cap));
    const int n_tiles = (L + 127) / 128;
    // Keys below lo are outside the window: the splits start at its first tile
    // (tile indices below are absolute).
    const int lo = kExt ? kv_window_lo(p, L) : 0;
    const int tile_begin = lo / 128 + split * p.split_tiles;
    const int tile_end = imin(tile_begin + p.split_tiles, n_tiles);
    const int T = tile_end - tile_begin;

    auto partial_row = [&](int n) -> int64_t {
        const int h = h_kv * p.G + n / nq;
        const int t = n % nq;
        return ((static_cast<int64_t>(b) * p.Hq + h) * nq + t) * p.num_splits + split;
    };

    if (T <= 0) {
        // A split with no key: O = 0 and lse2 = -inf for every query row.
        if (warp >= 2) {
            for (int idx = threadIdx.x - 64; idx < R * 32; idx += kSoftmaxThreads) {
                const int n = idx >> 5, c4 = idx & 31;
                if (p.direct_out) {
                    const int h = h_kv * p.G + n / nq, t = n % nq;
                    const int64_t orow = (static_cast<int64_t>(b) * nq + t) * p.Hq + h;
                    reinterpret_cast<uint2 *>(p.out + orow * 128)[c4] = make_uint2(0, 0);
                    if (c4 == 0 && p.lse) p.lse[(static_cast<int64_t>(b) * p.Hq + h) * nq + t] = -INFINITY;
                } else {
                    const int64_t row = partial_row(n);
                    reinterpret_cast<float4 *>(p.ws_o + row * 128)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (c4 == 0) p.ws_lse[row] = -INFINITY;
                }
            }
        }
        return;
    }

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::kBar);
    uint64_t *kv_full = bars;
    uint64_t *kv_empty = bars + kStagesD;
    uint64_t *q_full = bars + 2 * kStagesD;
    uint64_t *patch = q_full + 1;
    // S buffer (it & 1) is released by s_free: every softmax warp arrives there
    // once its read of S(it) has completed, early in the tile.
    uint64_t *s_full = q_full + 2;   // [2]
    uint64_t *p_full = q_full + 4;   // [2]
    uint64_t *pv_done = q_full + 6;  // [2]
    uint64_t *o_final = q_full + 8;
    uint64_t *vote_bar = q_full + 9;             // [column group][tile parity]: one arrival per warp
    uint64_t *xe_bar = vote_bar + 2 * Lay::kCG;  // [column group]: offsets posted for an O rescale
    uint64_t *s_free = xe_bar + Lay::kCG;        // [2]: S buffer read by every softmax warp
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::kMisc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + Lay::kMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesD; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(q_full, Lay::kSoftmaxWarps);
        mbar_init(patch, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], Lay::kSoftmaxWarps);
            mbar_init(&p_full[s], Lay::kSoftmaxWarps);
            mbar_init(&pv_done[s], 1);
        }
        mbar_init(o_final, 1);
        for (int g = 0; g < Lay::kCG; ++g) {
            mbar_init(&vote_bar[2 * g], 4);
            mbar_init(&vote_bar[2 * g + 1], 4);
            mbar_init(&xe_bar[g], 4);
        }
        // A status already set by another launch or CTA: unwind at once (every
        // wait returns false), decided once for the whole CTA.
        *abort_flag = (p.status && *reinterpret_cast<const volatile int32_t *>(p.status) != 0) ? 1u : 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Lay::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool last_partial = (L & 127) != 0 && tile_end == n_tiles;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const int nblk = kv_row_blocks<kExt>(p);
        PageLookup pl;
        int issued = 0;
        for (int it = 0; it < T; ++it) {
            const int tile = tile_begin + it;
            const int st = it % kStagesD;
            const uint32_t ph = (it / kStagesD) & 1;
            bool ok = wait_bar(&kv_empty[st], ph ^ 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            int row, blk;
            kv_tile_row<kExt>(p, b, h_kv, tile, pl, row, blk);
            if (lane == 0) {
                // An MXFP4 V tile lands unpacked (one byte per code in shared memory),
                // but the copy moves its packed bytes, half of the MXFP8 tile's.
                const int v_bytes = kExt && p.v_fp4 ? Lay::kVBytes / 2 : Lay::kVBytes;
                mbar_arrive_expect_tx(&kv_full[st], Lay::kKBytes + v_bytes + 1024);
                tma_load_3d(smem + Lay::kK + st * Lay::kKBytes, &tmap_k, 0, blk * 128, row, &kv_full[st]);
                tma_load_3d(smem + Lay::kV + st * Lay::kVBytes, &tmap_v, 0, 0, row * nblk + blk, &kv_full[st]);
                const int64_t atom = (static_cast<int64_t>(row) * nblk + blk) * 512;
                bulk_load(smem + Lay::kSfK + st * 512, p.k_scales + atom, 512, &kv_full[st]);
                bulk_load(smem + Lay::kSfV + st * 512, p.v_scales + atom, 512, &kv_full[st]);
            }
            issued = it + 1;
            if (last_partial && tile == tile_end - 1) {
                // Keys at or past L may hold anything (a reused cache); zero their
                // V codes and fully invalid V scale groups so no NaN reaches O.
                ok = wait_bar(&kv_full[st], ph, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) break;
                const int jv = L - tile * 128;
                uint8_t *vt = smem + Lay::kV + st * Lay::kVBytes;
                // (E2M1 has no NaN or infinity: MXFP4 V codes need no zeroing.)
                for (int c = lane; c < 128 * 8 && !(kExt && p.v_fp4); c += 32) {
                    const int row = c >> 3, q = c & 7;
                    if (16 * q + 16 <= jv) continue;
                    uint8_t *chunk = vt + row * 128 + ((q ^ (row & 7)) << 4);
                    for (int e = 0; e < 16; ++e)
                        if (16 * q + e >= jv) chunk[e] = 0;
                }
                uint8_t *sfv = smem + Lay::kSfV + st * 512;
                for (int row = lane; row < 128; row += 32)
                    for (int g = (jv + 31) / 32; g < 4; ++g) sfv[(row & 31) * 16 + (row >> 5) * 4 + g] = 0;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(patch);
            }
        }
        if (lane == 0) {
            for (int it = imax(0, issued - kStagesD); it < issued; ++it) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&kv_full[it % kStagesD], (it / kStagesD) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------------- MMA issuer
        // The whole warp runs the loop and waits, so the descriptors stay
        // warp-uniform; one elected lane issues the tcgen05 instructions.
        const bool leader = elect_one();
        bool ok = __all_sync(0xffffffffu, wait_bar(q_full, 0, abort_flag, p.status));
        if (ok) {
            tc_fence_after();
            const uint32_t sb = smem_u32(smem);
            constexpr uint32_t kIdQK = idesc_d(1u, NT);      // E2M1 x E2M1, N = NT
            // E4M3 V x E4M3 P, N = 2 NT; with MXFP4 V the A type field is E2M1 (5).
            const uint32_t kIdPV = idesc_d(0u, 2 * NT) | (kExt && p.v_fp4 ? (5u << 7) : 0u);
            // Descriptors for stage 0 / buffer 0; other stages are fixed
            // offsets of the 14-bit start-address field (in 16-byte units).
            const uint64_t dQ = smem_desc(sb + Lay::kQ, 16, 512, 4);
            const uint64_t dK0 = smem_desc(sb + Lay::kK, 16, 512, 4);
            const uint64_t dV0 = smem_desc(sb + Lay::kV, 16, 1024, 2);
            const uint64_t dP0 = smem_desc(sb + Lay::kP, 16, 1024, 2);
            const uint64_t dSfK0 = smem_desc(sb + Lay::kSfK, 0, 128, 0);
            const uint64_t dSfV0 = smem_desc(sb + Lay::kSfV, 0, 128, 0);
            const uint64_t dSfP0 = smem_desc(sb + Lay::kSfP, 0, 128, 0);
            if (leader) tc_cp_32x128b_warpx4(tmem + Lay::kColSfQ, smem_desc(sb + Lay::kSfQ, 0, 128, 0));
            const uint32_t tO = tmem + Lay::kColO;
            const uint32_t tSfQ = tmem + Lay::kColSfQ;
            auto issue_pv = [&](int j) -> bool {
                if (!__all_sync(0xffffffffu, wait_bar(&p_full[j & 1], (j >> 1) & 1, abort_flag, p.status)))
                    return false;
                tc_fence_after();
                const int st = j % kStagesD;
                const uint32_t tSfV = tmem + col_sf_v_d(NT, j & 1);
                const uint32_t tSfP = tmem + col_sf_p_d(NT, j & 1);
                const uint64_t dV = dV0 + static_cast<uint64_t>(st * (Lay::kVBytes >> 4));
                const uint64_t dP = dP0 + static_cast<uint64_t>((j & 1) * (Lay::kPBytes >> 4));
                if (leader) {
                    tc_cp_32x128b_warpx4(tSfV, dSfV0 + static_cast<uint64_t>(st * 32));
                    tc_cp_32x128b_warpx4(tSfP, dSfP0 + static_cast<uint64_t>((j & 1) * 32));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tO, dV + 2 * k, dP + 2 * k, sf_id_d(kIdPV, k), tSfV | (k << 30), tSfP | (k << 30),
                                    (j > 0 || k > 0) ? 1u : 0u);
                    tc_commit(&pv_done[j & 1]);
                    tc_commit(&kv_empty[st]);
                }
                __syncwarp();
                return true;
            };
            // S(it) = K(it) Q^T into S buffer it & 1, once K/V(it) have landed and
            // (from it = 2 on) every softmax warp has read S(it-2).
            auto issue_qk = [&](int it) -> bool {
                const int st = it % kStagesD;
                const int sbuf = it & 1;
                bool w = wait_bar(&kv_full[st], (it / kStagesD) & 1, abort_flag, p.status);
                if (w && last_partial && it == T - 1) w = wait_bar(patch, 0, abort_flag, p.status);
                if (w && it >= 2) w = wait_bar(&s_free[sbuf], ((it - 2) >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, w)) return false;
                tc_fence_after();
                const uint32_t tSfK = tmem + col_sf_k_d(NT, sbuf);
                const uint64_t dK = dK0 + static_cast<uint64_t>(st * (Lay::kKBytes >> 4));
                const uint32_t tS = tmem + static_cast<uint32_t>(NT * sbuf);
                if (leader) {
                    tc_cp_32x128b_warpx4(tSfK, dSfK0 + static_cast<uint64_t>(st * 32));
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc_mma_mxf4(tS, dK + 2 * kk, dQ + 2 * kk, sf_id_d(kIdQK, 2 * kk), tSfK | ((2u * kk) << 30),
                                    tSfQ | ((2u * kk) << 30), kk > 0 ? 1u : 0u);
                    tc_commit(&s_full[sbuf]);
                }
                __syncwarp();
                return true;
            };
            if (ST >= 5) {
                // Deep K/V pipeline: S(it+2) goes out as soon as S(it) has been read
                // (early in tile it), ahead of P V(it) (end of tile it), so the next
                // scores are ready when the softmax warps finish a tile.
                ok = issue_qk(0);
                if (ok && T > 1) ok = issue_qk(1);
                for (int it = 0; it < T && ok; ++it) {
                    if (it + 2 < T) ok = issue_qk(it + 2);
                    if (ok) ok = issue_pv(it);
                }
            } else {
                // Shallow pipeline: S(it) waits for K/V(it), which needs the stage that
                // P V(it - ST) frees, so P V goes first.
                for (int it = 0; it < T && ok; ++it) {
                    ok = issue_qk(it);
                    if (ok && it >= 1) ok = issue_pv(it - 1);
                }
                if (ok) ok = issue_pv(T - 1);
            }
            if (ok && leader) tc_commit(o_final);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax
        const int sw = warp - 2;
        const int quarter = warp & 3;     // TMEM lane quarter: tokens 32*quarter .. +31 of the tile
        const int cg = sw >> 2;           // column group: query rows c0 .. c0 + NC - 1
        const int c0 = cg * NC;
        const int nv = imax(0, imin(R - c0, NC));
        const int jt = quarter * 32 + lane;  // token within the tile, and channel in the epilogue
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int gbar = kBarGroup0 + cg;
        {
            // ------------------------------------------------------------ staging
            // Q^T operand: row n < R is query head h_kv*G + n/nq at token n%nq;
            // rows R..NT-1, and scale rows past NT, are zero.
            const int stid = threadIdx.x - 64;
            if (p.q_bf16) {
                // MXFP4-encode the bf16 query rows here, 16 lanes per row, with
                // the encoder of the quantization kernel (identical bytes).
                const int sub = lane & 15;
                for (int n0 = 2 * sw; n0 < NT; n0 += 2 * Lay::kSoftmaxWarps) {
                    const int n = n0 + (lane >> 4);
                    const bool valid = n < R;
                    uint4 raw = make_uint4(0, 0, 0, 0);
                    if (valid) {
                        const int h = h_kv * p.G + n / nq, t = n % nq;
                        raw = *reinterpret_cast<const uint4 *>(p.q_bf16 + b * p.q_sb + t * p.q_st + h * p.q_sh +
                                                               sub * 8);
                    }
                    int X;
                    const uint32_t packed = mxfp4_encode8(raw, valid, X);
                    const int j = sub >> 2;  // 16-byte chunk (block of 32 channels) of the 64-byte row
                    *reinterpret_cast<uint32_t *>(smem + Lay::kQ + n * 64 + ((j ^ ((n >> 1) & 3)) << 4) +
                                                  (sub & 3) * 4) = packed;
                    if ((sub & 3) == 0)
                        smem[Lay::kSfQ + (n & 31) * 16 + (n >> 5) * 4 + j] = valid ? static_cast<uint8_t>(X + 127) : 0;
                }
                for (int n = NT + stid; n < 128; n += kSoftmaxThreads)
                    *reinterpret_cast<uint32_t *>(smem + Lay::kSfQ + (n & 31) * 16 + (n >> 5) * 4) = 0;
            } else {
                for (int c = stid; c < NT * 4; c += kSoftmaxThreads) {
                    const int n = c >> 2, j = c & 3;
                    uint4 val = make_uint4(0, 0, 0, 0);
                    if (n < R) {
                        const int h = h_kv * p.G + n / nq, t = n % nq;
                        val = *reinterpret_cast<const uint4 *>(
                            p.q_codes + ((static_cast<int64_t>(b) * p.Hq + h) * p.q_cap + t) * 64 + j * 16);
                    }
                    *reinterpret_cast<uint4 *>(smem + Lay::kQ + n * 64 + ((j ^ ((n >> 1) & 3)) << 4)) = val;
                }
                for (int n = stid; n < 128; n += kSoftmaxThreads) {
                    uint32_t scw = 0;
                    if (n < R) {
                        const int h = h_kv * p.G + n / nq, t = n % nq;
                        scw = *reinterpret_cast<const uint32_t *>(
                            p.q_scales + ((static_cast<int64_t>(b) * p.Hq + h) * (p.q_cap / 128) + t / 128) * 512 +
                            (t & 31) * 16 + ((t & 127) >> 5) * 4);
                    }
                    *reinterpret_cast<uint32_t *>(smem + Lay::kSfQ + (n & 31) * 16 + (n >> 5) * 4) = scw;
                }
            }
            // P scale atoms start at 2^0 for P_hi rows [0, NT) and 2^-5 for P_lo rows
            // [NT, 2NT); the P^T buffers start at zero, and rows of absent queries
            // are never written again.
            for (int n = stid; n < 128; n += kSoftmaxThreads) {
                const uint32_t pw = n < NT ? kPhiScaleWord : kPloScaleWord;
                *reinterpret_cast<uint32_t *>(smem + Lay::kSfP + (n & 31) * 16 + (n >> 5) * 4) = pw;
                *reinterpret_cast<uint32_t *>(smem + Lay::kSfP + 512 + (n & 31) * 16 + (n >> 5) * 4) = pw;
            }
            for (int c = stid; c < 2 * Lay::kPBytes / 16; c += kSoftmaxThreads)
                reinterpret_cast<uint4 *>(smem + Lay::kP)[c] = make_uint4(0, 0, 0, 0);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && !p.test_stall) mbar_arrive(q_full);
        }
        // Exchange slots of this column group, [quarter][NC].
        float *xmax = reinterpret_cast<float *>(smem + Lay::kXmax) + cg * 4 * NC;
        int *xe = reinterpret_cast<int *>(smem + Lay::kXe) + cg * 4 * NC;
        float *lsum = reinterpret_cast<float *>(smem + Lay::kLsum) + cg * 4 * NC;
        int *esum = reinterpret_cast<int *>(smem + Lay::kEsum) + cg * 4 * NC;
        volatile uint32_t *votes = reinterpret_cast<volatile uint32_t *>(smem + Lay::kVote) + cg * 8;
        // Byte offset of (row c0 + i, token jt) in a P^T buffer is
        // pofs ^ ((i & 7) << 4) plus i * 128: the 128-byte swizzle puts token jt
        // of row n in 16-byte chunk (jt / 16) ^ (n % 8), and c0 is a multiple of 8.
        const int pofs = c0 * 128 + ((jt >> 4) << 4) + (jt & 15);
        const uint32_t pa_base = smem_u32(smem + Lay::kP) + static_cast<uint32_t>(pofs);
        // Per query row: -m, this warp's reference max (log2 units, so p =
        // 2^(s * scale - m)), kept in shared memory as it is the same for all
        // lanes; lacc, this thread's share of the row sum relative to m. Lane
        // i < NC also holds e_mine = m - m_O for row c0 + i, the exponent this
        // warp's scale byte gives its P block.
        float *m_neg = reinterpret_cast<float *>(smem + Lay::kMneg) + sw * NC;
        float lacc[NC];
#pragma unroll
        for (int i = 0; i < NC; ++i) lacc[i] = 0.f;
        if (lane < NC) m_neg[lane] = 0.f;
        __syncwarp();
        int e_mine = 0;
        uint32_t n_rescales = 0;
        const float sc = p.scale_log2;
        // Key bound of each query row: L, or L - nq + t + 1 for token t of a causal
        // verify block. Tabulated once so the per-tile loop needs no division.
        int *lim_s = reinterpret_cast<int *>(smem + Lay::kLim);
        if (sw == 0)
            for (int n = lane; n < NT; n += 32) lim_s[n] = p.causal ? imin(L, L - nq + (n % nq) + 1) : L;
        bar_sync(kBarAllSoftmax, kSoftmaxThreads);
        for (int it = 0; it < T; ++it) {
            const int sbuf = it & 1;
            bool ok = wait_bar(&s_full[sbuf], (it >> 1) & 1, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
            uint32_t sraw[NC];
            if (ok) {
                tc_fence_after();
                tmem_load_cols<NC>(tmem + lane_base + static_cast<uint32_t>(NT * sbuf + c0), sraw);
                tc_wait_ld();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sbuf]);  // the tensor core may now compute S(it+2)

            // u = s * scale - m (log2 units); -inf where the key is masked. Every row
            // may see this key unless it lies past L, or in the last nq-1 positions
            // where query t of the verify block stops at L - nq + t.
            const int tok = (tile_begin + it) * 128 + jt;
            float mrow[NC];
#pragma unroll
            for (int i = 0; i < NC; i += 4) {
                const float4 m4 = lds_f4(smem_u32(m_neg + i));
                mrow[i] = m4.x;
                mrow[i + 1] = m4.y;
                mrow[i + 2] = m4.z;
                mrow[i + 3] = m4.w;
            }
            // Rows past R (absent queries, zero Q) run through the same code with
            // s = 0; their results are never written.
            float u[NC];
#pragma unroll
            for (int i = 0; i < NC; i += 2) {
                const float2 v = ffma2(make_float2(__uint_as_float(sraw[i]), __uint_as_float(sraw[i + 1])),
                                       make_float2(sc, sc), make_float2(mrow[i], mrow[i + 1]));
                u[i] = v.x;
                u[i + 1] = v.y;
            }
            if (!(it > 0 && ok && tok < L - (p.causal ? nq - 1 : 0))) {
                // (Keys below the window's lo lie in the first tile of the first split.)
                const bool any_key = ok && tok < L && (!kExt || tok >= lo);
#pragma unroll
                for (int i = 0; i < NC; ++i)
                    if (!(any_key && tok < lim_s[c0 + i])) u[i] = -INFINITY;
            }
            if (it == 0) {
                // The group's first tile fixes m_O = m of each row: the row's largest
                // scaled score over the tile's 128 keys. A row with no key here has
                // no key in any later tile of the split (keys only grow), and keeps
                // m = 0 with a zero sum.
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    const float mx = warp_max_f32(u[i]);
                    if (lane == i) xmax[quarter * NC + i] = mx;
                }
                bar_sync(gbar, 128);
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    const float t = fmaxf(fmaxf(xmax[i], xmax[NC + i]), fmaxf(xmax[2 * NC + i], xmax[3 * NC + i]));
                    if (t > -INFINITY) {
                        if (lane == i) m_neg[i] = -t;
                        u[i] -= t;
                    }
                }
                __syncwarp();
            } else {
                // This warp's own moves: a row whose scores pass m by more than 2^kTauD
                // moves m up to the next whole binade above its maximum, so the offset
                // e in the scale byte stays an integer.
                float umax = u[0];
#pragma unroll
                for (int i = 1; i < NC; ++i) umax = fmaxf(umax, u[i]);
                if (__any_sync(0xffffffffu, umax > kTauD)) {
#pragma unroll
                    for (int i = 0; i < NC; ++i) {
                        const float mx = warp_max_f32(u[i]);
                        if (mx > kTauD) {
                            const float de = ceilf(fminf(mx, kMaxMoveD));
                            u[i] -= de;
                            const int dei = static_cast<int>(de);
                            lacc[i] *= exp2_neg_int(dei);
                            if (lane == i) {
                                m_neg[i] -= de;
                                e_mine += dei;
                            }
                        }
                    }
                    __syncwarp();
                }
            }
            // Post this warp's vote for the tile: bit 0, an offset past kEMaxD (O must
            // be rescaled before PV of this tile); bit 1, the CTA is unwinding.
            const bool over = __any_sync(0xffffffffu, lane < NC && e_mine > kEMaxD);
            if (lane == 0) {
                votes[sbuf * 4 + quarter] = (over ? 1u : 0u) | (*abort_flag ? 2u : 0u);
                mbar_arrive(&vote_bar[2 * cg + sbuf]);
            }
            // P buffer `sbuf` was last read by PV(it-2).
            if (it >= 2) {
                bool okw = wait_bar(&pv_done[sbuf], ((it >> 1) & 1) ^ 1, abort_flag, p.status);
                (void)__all_sync(0xffffffffu, okw);
            }
            // Encode P^T bytes from p as f16 pairs (rounding error 2^-11 of p, far
            // below what P_lo resolves): P_hi = E4M3(p); its value comes back
            // exactly as f16; P_lo = E4M3(32 (p - P_hi)), where the difference is
            // exact since P_hi is within 2^-4 of p. The row sums take p itself.
            const uint32_t pa = pa_base + static_cast<uint32_t>(sbuf * Lay::kPBytes);
            uint32_t hb[NC / 2], lb[NC / 2];
            const __half2 k32 = __float2half2_rn(32.f), km32 = __float2half2_rn(-32.f);
#pragma unroll
            for (int i = 0; i < NC; i += 2) {
                const float p0 = exp2_approx(u[i]);
                const float p1 = exp2_approx(u[i + 1]);
                const float2 la = fadd2(make_float2(lacc[i], lacc[i + 1]), make_float2(p0, p1));
                lacc[i] = la.x;
                lacc[i + 1] = la.y;
                const __half2 ph = __floats2half2_rn(p0, p1);
                const uint32_t phw = *reinterpret_cast<const uint32_t *>(&ph);
                const uint16_t h2 = cvt_e4m3x2_from_f16x2(phw);
                const uint32_t hvw = cvt_e4m3x2_to_f16x2(h2);
                const __half2 d = __hfma2(*reinterpret_cast<const __half2 *>(&hvw), km32, __hmul2(ph, k32));
                const uint16_t l2 = cvt_e4m3x2_from_f16x2(*reinterpret_cast<const uint32_t *>(&d));
                hb[i / 2] = h2;
                lb[i / 2] = l2;
            }
            StorePairs<NT, 0, NC>::run(pa, hb, lb);
            // Collect the vote. Every warp of the group reads the same four words.
            const bool okv = wait_bar_peers(&vote_bar[2 * cg + sbuf], (it >> 1) & 1);
            const uint32_t flags = okv ? (votes[sbuf * 4] | votes[sbuf * 4 + 1] | votes[sbuf * 4 + 2] |
                                          votes[sbuf * 4 + 3])
                                       : 2u;
            if (flags & 2u) break;
            if (flags & 1u) {
                // Some warp's offset passed kEMaxD: move m_O of each such row up by the
                // largest offset E among the group's warps. O (which holds PV up to
                // tile it-1) is scaled by 2^-E, every warp's offset drops by E, and
                // P bytes, being relative to each warp's own m, stay as they are.
                if (lane < NC) xe[quarter * NC + lane] = e_mine;
                __syncwarp();
                if (lane == 0) mbar_arrive(&xe_bar[cg]);
                const bool okx = wait_bar_peers(&xe_bar[cg], n_rescales & 1);
                ++n_rescales;
                int E = 0;
                if (okx && lane < NC) {
                    E = imax(imax(xe[lane], xe[NC + lane]), imax(xe[2 * NC + lane], xe[3 * NC + lane]));
                    if (E <= kEMaxD) E = 0;
                    e_mine -= E;
                }
                if (okx && it >= 1) {
                    bool okw = wait_bar(&pv_done[(it - 1) & 1], ((it - 1) >> 1) & 1, abort_flag, p.status);
                    if (__all_sync(0xffffffffu, okw)) {
                        tc_fence_after();
                        rescale_o_cols(tmem + lane_base + Lay::kColO + c0, NT, NC, E);
                    }
                }
            }
            // Scale bytes of this warp's key block (byte `quarter`) in the buffer's
            // atom: row c0+i (P_hi) gets 2^e, row NT+c0+i (P_lo) 2^(e-5). An offset
            // far below m_O clamps at the smallest E8M0 value; such a block is
            // negligible against the row's maximum.
            if (lane < NC) {
                uint8_t *atom = smem + Lay::kSfP + sbuf * 512;
                const int n = c0 + lane, nl = NT + c0 + lane;
                atom[(n & 31) * 16 + (n >> 5) * 4 + quarter] = static_cast<uint8_t>(imax(0, 127 + e_mine));
                atom[(nl & 31) * 16 + (nl >> 5) * 4 + quarter] = static_cast<uint8_t>(imax(0, 122 + e_mine));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[sbuf]);
        }
        // ----------------------------------------------------------------- epilogue
        bool ok = !*abort_flag;
        if (ok) ok = wait_bar(o_final, 0, abort_flag, p.status);
        ok = __all_sync(0xffffffffu, ok);
        // Row sums: over this warp's lanes, then over the group's four warps, each
        // scaled from its own m to m_O by 2^e.
#pragma unroll
        for (int i = 0; i < NC; ++i) {
            float v = lacc[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) lsum[quarter * NC + i] = v;
        }
        if (lane < NC) esum[quarter * NC + lane] = e_mine;
        bar_sync(gbar, 128);
        if (ok && !*abort_flag) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < NC; c += 4) {
                if (c >= nv) break;
                uint32_t ohi[4], olo[4];
                tmem_load_cols<4>(tmem + lane_base + Lay::kColO + c0 + c, ohi);
                tmem_load_cols<4>(tmem + lane_base + Lay::kColO + NT + c0 + c, olo);
                tc_wait_ld();
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = c + e;
                    if (i >= nv) break;
                    float l = 0.f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) l += ldexpf(lsum[q * NC + i], esum[q * NC + i]);
                    const bool any = l > 0.f;
                    // O and l are both relative to m_O = m - e.
                    const float o = any ? (__uint_as_float(ohi[e]) + __uint_as_float(olo[e])) / l : 0.f;
                    const float lse2 =
                        any ? log2f(l) - m_neg[i] - static_cast<float>(esum[quarter * NC + i]) : -INFINITY;
                    if (p.direct_out) {
                        const int n = c0 + i, h = h_kv * p.G + n / nq, t = n % nq;
                        p.out[((static_cast<int64_t>(b) * nq + t) * p.Hq + h) * 128 + jt] = __float2bfloat16_rn(o);
                        if (jt == 0 && p.lse)
                            p.lse[(static_cast<int64_t>(b) * p.Hq + h) * nq + t] =
                                any ? lse2 * 0.6931471805599453f : -INFINITY;
                    } else {
                        const int64_t row = partial_row(c0 + i);
                        p.ws_o[row * 128 + jt] = o;
                        if (jt == 0) p.ws_lse[row] = lse2;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::kTmemCols);
    }
}

template <int NT, int RW, int NC, int ST, int MINB>
static cudaError_t launch_nt(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, int grid,
                             cudaStream_t stream) {
    using Lay = DecodeLayout<NT, RW, NC, ST>;
    static_assert(MINB * (Lay::kBytes + kSmemReservedPerCta) <= kSmemPerSm, "MINB CTAs per SM must fit");
    constexpr int kMaxDevices = 64;
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !configured[dev]) {
        e = cudaFuncSetAttribute(qk4v8_decode_kernel<NT, RW, NC, ST, MINB, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kBytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(qk4v8_decode_kernel<NT, RW, NC, ST, MINB, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kBytes);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) configured[dev] = true;
    }
    if (p.window > 0 || p.block_table || p.v_fp4)
        qk4v8_decode_kernel<NT, RW, NC, ST, MINB, true><<<grid, Lay::kThreads, Lay::kBytes, stream>>>(tk, tv, p);
    else
        qk4v8_decode_kernel<NT, RW, NC, ST, MINB, false><<<grid, Lay::kThreads, Lay::kBytes, stream>>>(tk, tv, p);
    return cudaGetLastError();
}

cudaError_t launch_decode(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, int grid,
                          cudaStream_t stream) {
    const int R = p.G * p.Sq;
    if (R <= 4) return launch_nt<16, 4, 4, kDecodeStages8, 2>(tk, tv, p, grid, stream);
    if (R <= 8) return launch_nt<16, 8, 8, kDecodeStages8, 2>(tk, tv, p, grid, stream);
    if (R <= 16) return launch_nt<16, 16, 16, kDecodeStages16, 2>(tk, tv, p, grid, stream);
    if (R <= 32) return launch_nt<32, 32, 16, 6, 1>(tk, tv, p, grid, stream);
    return launch_nt<64, 64, 16, 6, 1>(tk, tv, p, grid, stream);
}

}  // namespace qk4v8
