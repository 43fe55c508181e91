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
//     The owner of the next tile learns E through a one-way handshake
//     posted at the end of each tile, and m_O through one posted early in the
//     unit's first tile.
// P is kept as two E4M3 terms with the same scales: P_hi = E4M3(p) and
// P_lo = E4M3(p - P_hi), about 8 significant bits. V carries an extra row of
// ones, so O column 128 accumulates the softmax denominator sum(P_hi + P_lo)
// in the same MMAs.
//
// Warp roles (352 threads): warps 0..7 softmax and epilogue, warp 8 Q/K
// producer (TMA), warp 9 TMEM allocator and MMA issuer, warp 10 V producer
// (TMA). The producers and the MMA issuer each run on one elected thread.
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
#include "tile_ops.cuh"

namespace qk4v8 {

namespace {

constexpr int kPfKStages = 6;               // K tiles in flight (freed when QK^T of the tile completes)
constexpr int kPfVStages = 4;               // V tiles in flight (freed when P V of the tile completes)
constexpr int kPfSoftmaxWarps = 8;          // two per TMEM lane quarter, alternate key tiles
// Warps 0..7 softmax, then the Q/K producer, the MMA issuer and the V producer.
constexpr int kPfThreads = 32 * kPfSoftmaxWarps + 96;
constexpr int kPfProducerWarp = 8;          // Q and K tiles with their scales
constexpr int kPfMmaWarp = 9;
constexpr int kPfVWarp = 10;                // V tiles with their scales
constexpr float kPfTau = 8.0f;              // m_w moves once a score passes it by 2^8
constexpr int kPfEMax = 64;                 // largest e = m_w - m_O before O is rescaled
constexpr float kPfMaxMove = 16777216.0f;   // cap on one move of m_w, keeps it an exact integer

// Shared memory map (byte offsets from a 1024-aligned base).
struct PfSmem {
    static constexpr int kQBytes = 128 * 64;
    static constexpr int kQ = 0;                                   // 2 buffers: 128 rows x 64 B, 64-byte swizzle
    static constexpr int kKBytes = 128 * 64;
    static constexpr int kK = kQ + 2 * kQBytes;                    // per stage: 128 keys x 64 B
    static constexpr int kVRows = 144;                             // 128 channels, ones row, 15 zero rows
    static constexpr int kVBytes = kVRows * 128;
    static constexpr int kVTmaBytes = 128 * 128;
    static constexpr int kV = kK + kPfKStages * kKBytes;           // per stage: 144 rows x 128 B, 128-byte swizzle
    static constexpr int kPBuf = 2 * 128 * 128;                    // P_hi then P_lo, 128 rows x 128 B each
    static constexpr int kP = kV + kPfVStages * kVBytes;           // 2 buffers, one per warp parity
    static constexpr int kSfQ = kP + 2 * kPBuf;                    // 512-byte scale atoms: 2 Q buffers
    static constexpr int kSfK = kSfQ + 2 * 512;
    static constexpr int kSfV = kSfK + kPfKStages * 512;
    static constexpr int kSfP = kSfV + kPfVStages * 512;           // one atom per P buffer (P_hi and P_lo share it)
    static constexpr int kSfOne = kSfP + 2 * 512;
    // Handshake slots [quarter][tile parity][row (lane)]: the shift E of O, and
    // (tile parity 0 only) the reference m_O.
    static constexpr int kHsE = kSfOne + 512;                      // int [4][2][32]
    static constexpr int kHsM = kHsE + 4 * 2 * 32 * 4;             // float [4][2][32]
    // QK stage: row maxima [unit slot][warp parity][128] and arrival counters
    // [quarter][unit slot]; 8 unit slots, more than one parity can lead the other.
    static constexpr int kXmax = kHsM + 4 * 2 * 32 * 4;
    static constexpr int kXcnt = kXmax + 8 * 2 * 128 * 4;
    static constexpr int kBar = kXcnt + 4 * 8 * 4;
    // k_full/k_empty, v_full/v_empty per stage; q_full/q_empty per Q buffer;
    // patch; s_full, s_free, p_full, pv_done per parity; o_full, o_free, drain;
    // handshake [4 quarters][2]; m_O handshake [4 quarters]; unit end [4 quarters].
    static constexpr int kNumBars = 2 * kPfKStages + 2 * kPfVStages + 4 + 1 + 8 + 3 + 8 + 4 + 4;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kUsed = kMisc + 16;
    static constexpr int kBytes = kUsed + 1024;  // slack for aligning the base
};
static_assert(PfSmem::kK % 1024 == 0 && PfSmem::kV % 1024 == 0 && PfSmem::kP % 1024 == 0 &&
                  PfSmem::kVBytes % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
static_assert(PfSmem::kBar % 8 == 0, "mbarrier alignment");
static_assert(PfSmem::kBytes <= 227 * 1024, "shared memory budget");

// TMEM columns (512 allocated, one CTA per SM).
constexpr uint32_t kPfTmemCols = 512;
constexpr uint32_t kPfColO = 256;  // 144 columns: O[:, 0:128], the row sum in column 128
__device__ __forceinline__ uint32_t pf_col_s(int buf) { return 128u * buf; }
__device__ __forceinline__ uint32_t pf_col_sf_q(int buf) { return 400u + 4u * buf; }
__device__ __forceinline__ uint32_t pf_col_sf_k(int buf) { return 408u + 4u * buf; }
// V scales per buffer: 4 columns, then 4 constant columns for the ones row.
__device__ __forceinline__ uint32_t pf_col_sf_v(int buf) { return 416u + 8u * buf; }
__device__ __forceinline__ uint32_t pf_col_sf_p(int buf) { return 432u + 4u * buf; }

constexpr uint32_t pf_idesc(uint32_t fmt, uint32_t n) {
    return (fmt << 7) | (fmt << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}
constexpr uint32_t kPfIdQK = pf_idesc(1u, 128);             // E2M1 x E2M1, N = 128 keys
constexpr uint32_t kPfIdPV = pf_idesc(0u, PfSmem::kVRows);  // E4M3 x E4M3, N = 144
__device__ __forceinline__ uint32_t pf_sf_id(uint32_t idesc, uint32_t id) { return idesc | (id << 29) | (id << 4); }

struct PfUnit {
    int b, h_q, h_kv, q0, L, T;
};

// Integer quotient a / b for 0 <= a, 1 <= b through the float reciprocal rb of
// b, corrected to the exact value by the integer remainder. A unit's
// description is worked out on the issue paths of the producer and the MMA
// warp at every unit change, where the emulated integer divisions cost
// hundreds of cycles.
__device__ __forceinline__ int pf_div(int a, int b, float rb) {
    int q = static_cast<int>(static_cast<float>(a) * rb);
    int r = a - q * b;
    while (r < 0) {
        --q;
        r += b;
    }
    while (r >= b) {
        ++q;
        r -= b;
    }
    return q;
}

struct PfDecode {
    int per;           // units per query tile row: B * Hq
    float r_per, r_hq, r_g;
};

__device__ __forceinline__ PfDecode pf_decode(const AttnParams &p) {
    PfDecode d;
    d.per = p.B * p.Hq;
    d.r_per = 1.0f / static_cast<float>(d.per);
    d.r_hq = 1.0f / static_cast<float>(p.Hq);
    d.r_g = 1.0f / static_cast<float>(p.G);
    return d;
}

// Work unit `idx`: one query head and 128 query tokens. Units are numbered
// longest first (the last query tiles of a causal prefill see the most keys).
__device__ __forceinline__ PfUnit pf_unit(const AttnParams &p, const PfDecode &d, int idx) {
    PfUnit u;
    const int row = pf_div(idx, d.per, d.r_per);
    const int qt = p.n_qtiles - 1 - row;
    const int rem = idx - row * d.per;
    u.b = pf_div(rem, p.Hq, d.r_hq);
    u.h_q = rem - u.b * p.Hq;
    u.h_kv = pf_div(u.h_q, p.G, d.r_g);
    u.q0 = qt * 128;
    const int R = imin(128, p.Sq - u.q0);
    const int L = p.seqlens ? p.seqlens[u.b] : p.Lk;
    u.L = imax(0, imin(L, p.kv_cap));
    int kv_end = u.L;
    if (p.causal) kv_end = imin(u.L, u.q0 + R + u.L - p.Sq);
    u.T = kv_end > 0 ? (kv_end + 127) >> 7 : 0;
    return u;
}

}  // namespace

template <bool kStageQK>
__global__ void __launch_bounds__(kPfThreads, 1)
    qk4v8_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const AttnParams p) {
    using S = PfSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_units = p.B * p.Hq * p.n_qtiles;
    const PfDecode dc = pf_decode(p);

    // Softmax thread identity (warps 0..7): lane quarter, warp parity, row in the tile.
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int pp = warp >> 2;      // the warp owns the tiles whose global index has parity pp
    const int row = quarter * 32 + lane;
    // Output channels this warp writes in the epilogue: 64 per parity.
    const int c_lo = 64 * pp;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::kBar);
    uint64_t *k_full = bars;
    uint64_t *k_empty = k_full + kPfKStages;
    uint64_t *v_full = k_empty + kPfKStages;
    uint64_t *v_empty = v_full + kPfVStages;
    uint64_t *q_full = v_empty + kPfVStages;  // [Q buffer]
    uint64_t *q_empty = q_full + 2;           // [Q buffer]
    uint64_t *patch = q_empty + 2;
    uint64_t *s_full = patch + 1;    // [parity]
    uint64_t *s_free = s_full + 2;   // [parity]
    uint64_t *p_full = s_free + 2;   // [parity]
    uint64_t *pv_done = p_full + 2;  // [parity]
    uint64_t *o_full = pv_done + 2;
    uint64_t *o_free = o_full + 1;
    uint64_t *drain = o_free + 1;
    uint64_t *hs_bar = drain + 1;    // [quarter][parity]
    uint64_t *mo_bar = hs_bar + 8;   // [quarter]
    uint64_t *ue_bar = mo_bar + 4;   // [quarter]: both warps of the quarter are done with a unit
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
        for (int s = 0; s < 2; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], 4);
            mbar_init(&p_full[s], 4);
            mbar_init(&pv_done[s], 1);
        }
        mbar_init(patch, 1);
        mbar_init(o_full, 1);
        mbar_init(o_free, kPfSoftmaxWarps);
        mbar_init(drain, 1);
        for (int g = 0; g < 8; ++g) mbar_init(&hs_bar[g], 1);
        for (int g = 0; g < 4; ++g) {
            mbar_init(&mo_bar[g], 1);
            mbar_init(&ue_bar[g], 2);
        }
        if (kStageQK)
            for (int i = 0; i < 4 * 8; ++i) reinterpret_cast<int *>(smem + S::kXcnt)[i] = 0;
        // A status already set by another launch or CTA: unwind at once (every
        // wait returns false), uniformly for the whole CTA.
        *abort_flag = (p.status && *reinterpret_cast<const volatile int32_t *>(p.status) != 0) ? 1u : 0u;
        fence_barrier_init();
    }
    if (warp == kPfMmaWarp) {
        tmem_alloc(tmem_slot, kPfTmemCols);
        tmem_relinquish();
    }
    if (!kStageQK && warp == kPfVWarp) {
        // Constant V rows: row 128 = 1.0 (E4M3 0x38), rows 129..143 = 0, and a
        // scale atom of 2^0 for them. TMA never writes these rows.
        for (int s = 0; s < kPfVStages; ++s)
            for (int cc = lane; cc < 16 * 8; cc += 32) {
                const int r = 128 + (cc >> 3);
                const uint32_t fillv = r == 128 ? 0x38383838u : 0u;
                *reinterpret_cast<uint4 *>(smem + S::kV + s * S::kVBytes + r * 128 + (cc & 7) * 16) =
                    make_uint4(fillv, fillv, fillv, fillv);
            }
        reinterpret_cast<uint4 *>(smem + S::kSfOne)[lane] = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kPfProducerWarp) {
        // ----------------------------------------------------------- Q/K producer
        // One elected thread: each step is a probe of one barrier and three copy
        // instructions, and this thread's pace bounds the QK^T stage's.
        uint32_t pred;
        asm volatile(
            "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.u32 %0, 1, 0, e;\n\t}"
            : "=r"(pred));
        if (pred != 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            const int nblk = p.kv_cap / 128;
            int g = 0, c = 0;  // tiles and units so far (units with at least one tile)
            int gk_issued = 0, q_issued = 0;  // copies issued (global tile / unit counts)
            bool ok = true;
            for (int un = blockIdx.x; un < n_units && ok; un += gridDim.x) {
                const PfUnit u = pf_unit(p, dc, un);
                const int T = u.T;
                if (T <= 0) continue;
                const int kvh = u.b * p.Hkv + u.h_kv;
                const int qb = c & 1;
                // Q of this unit (TMA; rows past Sq are padding in the packed format)
                // and its scale atom. The MMA warp frees the buffer after the unit's
                // last QK^T.
                const uint32_t qpar = ((c >> 1) & 1) ^ 1;
                ok = mbar_test_wait(&q_empty[qb], qpar) || wait_bar(&q_empty[qb], qpar, abort_flag, p.status);
                if (!ok) break;
                if (!(p.test_stall && c == 0)) {
                    const int qhead = u.b * p.Hq + u.h_q;
                    mbar_arrive_expect_tx(&q_full[qb], S::kQBytes + 512);
                    tma_load_3d(smem + S::kQ + qb * S::kQBytes, &tmap_q, 0, u.q0, qhead, &q_full[qb]);
                    bulk_load(smem + S::kSfQ + qb * 512,
                              p.q_scales + (static_cast<int64_t>(qhead) * (p.q_cap / 128) + u.q0 / 128) * 512, 512,
                              &q_full[qb]);
                    q_issued = c + 1;
                }
                // K tiles: the ring frees as soon as QK^T of a tile completes.
                for (int it = 0; it < T; ++it) {
                    const int gk = g + it;
                    const int st = gk % kPfKStages;
                    const uint32_t kpar = ((gk / kPfKStages) & 1) ^ 1;
                    ok = mbar_test_wait(&k_empty[st], kpar) || wait_bar(&k_empty[st], kpar, abort_flag, p.status);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&k_full[st], S::kKBytes + 512);
                    tma_load_3d(smem + S::kK + st * S::kKBytes, &tmap_k, 0, it * 128, kvh, &k_full[st]);
                    bulk_load(smem + S::kSfK + st * 512, p.k_scales + (static_cast<int64_t>(kvh) * nblk + it) * 512,
                              512, &k_full[st]);
                    gk_issued = gk + 1;
                }
                g += T;
                ++c;
            }
            // Let every issued copy land before the CTA can retire.
            auto settle = [&](uint64_t *bar, uint32_t parity) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(bar, parity))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            };
            for (int gk = imax(0, gk_issued - kPfKStages); gk < gk_issued; ++gk)
                settle(&k_full[gk % kPfKStages], (gk / kPfKStages) & 1);
            for (int cq = imax(0, q_issued - 2); cq < q_issued; ++cq) settle(&q_full[cq & 1], (cq >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == kPfVWarp) {
        // ------------------------------------------------------------- V producer
        // One elected thread, like the Q/K producer: a whole warp waiting here
        // takes issue slots from the softmax warps that share its scheduler.
        uint32_t pred;
        asm volatile(
            "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.u32 %0, 1, 0, e;\n\t}"
            : "=r"(pred));
        if (!kStageQK && pred != 0) {
            prefetch_tensormap(&tmap_v);
            const int nblk = p.kv_cap / 128;
            int g = 0;
            int gv_issued = 0;
            bool ok = true;
            for (int un = blockIdx.x; un < n_units && ok; un += gridDim.x) {
                const PfUnit u = pf_unit(p, dc, un);
                const int T = u.T;
                if (T <= 0) continue;
                const int kvh = u.b * p.Hkv + u.h_kv;
                const bool last_partial = (u.L & 127) != 0 && T == (u.L + 127) / 128;
                // V tiles: the ring frees only after P V of a tile.
                for (int jt = 0; jt < T && ok; ++jt) {
                    const int gv = g + jt;
                    const int sv = gv % kPfVStages;
                    const uint32_t ph = (gv / kPfVStages) & 1;
                    ok = mbar_test_wait(&v_empty[sv], ph ^ 1) || wait_bar(&v_empty[sv], ph ^ 1, abort_flag, p.status);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&v_full[sv], S::kVTmaBytes + 512);
                    tma_load_3d(smem + S::kV + sv * S::kVBytes, &tmap_v, 0, 0, kvh * nblk + jt, &v_full[sv]);
                    bulk_load(smem + S::kSfV + sv * 512, p.v_scales + (static_cast<int64_t>(kvh) * nblk + jt) * 512,
                              512, &v_full[sv]);
                    gv_issued = gv + 1;
                    if (last_partial && jt == T - 1) {
                        // Keys at or past L may hold anything (a reused buffer). Their P
                        // is zero, but a NaN code or scale in V would still poison O:
                        // zero them once the tile has landed, and tell the MMA warp.
                        ok = wait_bar(&v_full[sv], ph, abort_flag, p.status);
                        if (!ok) break;
                        const int jv = u.L - jt * 128;  // valid keys in this tile, 1..127
                        uint8_t *vt = smem + S::kV + sv * S::kVBytes;
                        const int q0 = jv >> 4;  // 16-byte chunk (of each channel row) holding key jv
                        for (int r = 0; r < 128; ++r) {
                            for (int q = q0; q < 8; ++q) {
                                uint8_t *chunk = vt + r * 128 + ((q ^ (r & 7)) << 4);
                                if (16 * q >= jv) {
                                    *reinterpret_cast<uint4 *>(chunk) = make_uint4(0, 0, 0, 0);
                                } else {
                                    for (int e = jv - 16 * q; e < 16; ++e) chunk[e] = 0;
                                }
                            }
                        }
                        uint8_t *sfv = smem + S::kSfV + sv * 512;
                        for (int r = 0; r < 128; ++r)
                            for (int gq = (jv + 31) / 32; gq < 4; ++gq) sfv[(r & 31) * 16 + (r >> 5) * 4 + gq] = 0;
                        fence_proxy_async_smem();
                        mbar_arrive(patch);
                    }
                }
                g += T;
            }
            // Let every issued copy land before the CTA can retire.
            for (int gv = imax(0, gv_issued - kPfVStages); gv < gv_issued; ++gv) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&v_full[gv % kPfVStages], (gv / kPfVStages) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
        }
        __syncwarp();
    } else if (warp == kPfMmaWarp) {
        // -------------------------------------------------------------- MMA issuer
        // Every tcgen05 instruction of this role (copies of scale atoms, MMAs,
        // commits) is issued by a single thread, so one elected thread runs the
        // whole loop: its waits need no warp votes and its issue path no
        // reconvergence. That path sets the pace of the QK^T stage.
        uint32_t pred;
        asm volatile(
            "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.u32 %0, 1, 0, e;\n\t}"
            : "=r"(pred));
        if (pred != 0) {
            const uint32_t sb = smem_u32(smem);
            // Descriptors for stage / buffer 0; the others are fixed offsets of the
            // 14-bit start-address field (16-byte units).
            const uint64_t dQ0 = smem_desc(sb + S::kQ, 16, 512, 4);
            const uint64_t dK0 = smem_desc(sb + S::kK, 16, 512, 4);
            const uint64_t dV0 = smem_desc(sb + S::kV, 16, 1024, 2);
            const uint64_t dP0 = smem_desc(sb + S::kP, 16, 1024, 2);
            const uint64_t dSfQ0 = smem_desc(sb + S::kSfQ, 0, 128, 0);
            const uint64_t dSfK0 = smem_desc(sb + S::kSfK, 0, 128, 0);
            const uint64_t dSfV0 = smem_desc(sb + S::kSfV, 0, 128, 0);
            const uint64_t dSfP0 = smem_desc(sb + S::kSfP, 0, 128, 0);
            const uint32_t tO = tmem + kPfColO;
            bool ok = true;
            if (!kStageQK) {
                // The ones row's scale, for both V scale buffers, once.
                const uint64_t dOne = smem_desc(sb + S::kSfOne, 0, 128, 0);
                tc_cp_32x128b_warpx4(tmem + pf_col_sf_v(0) + 4, dOne);
                tc_cp_32x128b_warpx4(tmem + pf_col_sf_v(1) + 4, dOne);
            }
            int g = 0, c = 0, n_patch = 0;
            // The next unit's description is worked out while this unit's first S
            // computes, off the issue path of the unit transition.
            PfUnit nu = pf_unit(p, dc, blockIdx.x);
            for (int un = blockIdx.x; un < n_units && ok; un += gridDim.x) {
                const PfUnit u = nu;
                const int T = u.T;
                if (T <= 0) {
                    if (un + static_cast<int>(gridDim.x) < n_units) nu = pf_unit(p, dc, un + gridDim.x);
                    continue;
                }
                const int qb = c & 1;
                const bool last_partial = !kStageQK && (u.L & 127) != 0 && T == (u.L + 127) / 128;
                ok = mbar_test_wait(&q_full[qb], (c >> 1) & 1) ||
                     wait_bar(&q_full[qb], (c >> 1) & 1, abort_flag, p.status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t tSfQ = tmem + pf_col_sf_q(qb);
                const uint64_t dQ = dQ0 + static_cast<uint64_t>(qb * (S::kQBytes >> 4));
                tc_cp_32x128b_warpx4(tSfQ, dSfQ0 + static_cast<uint64_t>(qb * 32));
                // S(gi) = Q K(gi)^T into S buffer gi & 1, once K(gi) has landed and the
                // warps of parity gi & 1 have read S(gi-2) out of that buffer.
                auto issue_qk = [&](int i) -> bool {
                    const int gi = g + i;
                    const int st = gi % kPfKStages;
                    const uint32_t kpar = (gi / kPfKStages) & 1;
                    const uint32_t spar = ((gi - 2) >> 1) & 1;
                    // Both inputs are usually ready by now: one probe of the two
                    // barriers, the bounded waits only when it fails.
                    bool w = gi >= 2 ? mbar_test_wait2(&k_full[st], kpar, &s_free[gi & 1], spar)
                                     : mbar_test_wait(&k_full[st], kpar);
                    if (!w) {
                        w = wait_bar(&k_full[st], kpar, abort_flag, p.status);
                        if (w && gi >= 2) w = wait_bar(&s_free[gi & 1], spar, abort_flag, p.status);
                    }
                    if (!w) return false;
                    tc_fence_after();
                    const uint32_t tSfK = tmem + pf_col_sf_k(gi & 1);
                    const uint64_t dK = dK0 + static_cast<uint64_t>(st * (S::kKBytes >> 4));
                    const uint32_t tS = tmem + pf_col_s(gi & 1);
                    tc_cp_32x128b_warpx4(tSfK, dSfK0 + static_cast<uint64_t>(st * 32));
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc_mma_mxf4(tS, dQ + 2 * kk, dK + 2 * kk, pf_sf_id(kPfIdQK, 2 * kk), tSfQ | ((2u * kk) << 30),
                                    tSfK | ((2u * kk) << 30), kk > 0 ? 1u : 0u);
                    tc_commit(&s_full[gi & 1]);
                    tc_commit(&k_empty[st]);
                    return true;
                };
                // O += P(gi) V(gi), once V(gi) has landed and the warps of parity gi & 1
                // have written P(gi); the unit's first one overwrites O, once the
                // previous unit's epilogue has read it.
                auto issue_pv = [&](int i) -> bool {
                    const int gi = g + i;
                    const int sv = gi % kPfVStages;
                    const uint32_t vpar = (gi / kPfVStages) & 1;
                    const uint32_t ppar = (gi >> 1) & 1;
                    const bool need_patch = last_partial && i == T - 1;
                    const bool need_ofree = i == 0 && c >= 1;
                    bool w = !need_patch && !need_ofree && mbar_test_wait2(&v_full[sv], vpar, &p_full[gi & 1], ppar);
                    if (!w) {
                        w = wait_bar(&v_full[sv], vpar, abort_flag, p.status);
                        if (w && need_patch) w = wait_bar(patch, n_patch & 1, abort_flag, p.status);
                        if (w && need_ofree) w = wait_bar(o_free, (c - 1) & 1, abort_flag, p.status);
                        if (w) w = wait_bar(&p_full[gi & 1], ppar, abort_flag, p.status);
                    }
                    if (!w) return false;
                    tc_fence_after();
                    const uint32_t tSfV = tmem + pf_col_sf_v(gi & 1);
                    const uint32_t tSfP = tmem + pf_col_sf_p(gi & 1);
                    const uint64_t dV = dV0 + static_cast<uint64_t>(sv * (S::kVBytes >> 4));
                    const uint64_t dPhi = dP0 + static_cast<uint64_t>((gi & 1) * (S::kPBuf >> 4));
                    const uint64_t dPlo = dPhi + static_cast<uint64_t>((128 * 128) >> 4);
                    tc_cp_32x128b_warpx4(tSfV, dSfV0 + static_cast<uint64_t>(sv * 32));
                    tc_cp_32x128b_warpx4(tSfP, dSfP0 + static_cast<uint64_t>((gi & 1) * 32));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tO, dPhi + 2 * k, dV + 2 * k, pf_sf_id(kPfIdPV, k), tSfP | (k << 30),
                                    tSfV | (k << 30), (i > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tO, dPlo + 2 * k, dV + 2 * k, pf_sf_id(kPfIdPV, k), tSfP | (k << 30),
                                    tSfV | (k << 30), 1u);
                    tc_commit(&pv_done[gi & 1]);
                    tc_commit(&v_empty[sv]);
                    return true;
                };
                // The tensor pipe runs in issue order, so the issue order follows the
                // order in which the softmax warps release their inputs: S(i) is read
                // early in tile i, while P(i-1) is written at the end of tile i-1 by the
                // other warp, later. So: S(0), S(1), then per tile i: S(i+2) once S(i)
                // has been read, then P(i-1) V(i-1). S(i+2) then never queues behind a
                // P V.
                ok = issue_qk(0);
                if (ok && T > 1) ok = issue_qk(1);
                if (un + static_cast<int>(gridDim.x) < n_units) nu = pf_unit(p, dc, un + gridDim.x);
                for (int i = 0; i < T && ok; ++i) {
                    if (i + 2 < T) ok = issue_qk(i + 2);
                    if (ok && !kStageQK && i >= 1) ok = issue_pv(i - 1);
                }
                if (ok && !kStageQK) ok = issue_pv(T - 1);
                if (!ok) break;
                tc_commit(&q_empty[qb]);  // Q buffer and its scale columns free for unit c + 2
                if (!kStageQK) tc_commit(o_full);
                if (last_partial) ++n_patch;
                g += T;
                ++c;
            }
            // Every tcgen05 operation issued above has completed once `drain` does,
            // also when the loop unwound early, so TMEM is freed with nothing in
            // flight.
            tc_commit(drain);
        }
        __syncwarp();
        (void)wait_peers(drain, 0);
    } else if (warp < kPfSoftmaxWarps) {
        // ------------------------------------------------------------------ softmax
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        // Handshake slots of this thread's row (shared-space addresses), E and m
        // by tile parity.
        const uint32_t a_e = smem_u32(smem + S::kHsE) + quarter * 256 + lane * 4;
        const uint32_t a_m = smem_u32(smem + S::kHsM) + quarter * 256 + lane * 4;
        uint64_t *hs = hs_bar + quarter * 2;
        uint8_t *pbuf = smem + S::kP + pp * S::kPBuf;
        float *xmax = reinterpret_cast<float *>(smem + S::kXmax);
        int *xcnt = reinterpret_cast<int *>(smem + S::kXcnt);
        const int swz = row & 7;
        const float sc = p.scale_log2;
        int g = 0, c = 0;  // tiles and units so far (units with at least one tile)
        bool ok = true;
        for (int un = blockIdx.x; un < n_units && ok; un += gridDim.x) {
            const PfUnit u = pf_unit(p, dc, un);
            const int T = u.T;
            const int qi = u.q0 + row;
            const bool row_valid = qi < p.Sq;
            if (T <= 0) {
                // No key for any row of the tile: O = 0, lse = -inf.
                if (row_valid && !kStageQK) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        p.out + ((static_cast<int64_t>(u.b) * p.Sq + qi) * p.Hq + u.h_q) * 128 + c_lo);
#pragma unroll
                    for (int q = 0; q < 8; ++q) dst[q] = make_uint4(0, 0, 0, 0);
                }
                if (row_valid && pp == 0 && p.lse)
                    p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] = -INFINITY;
                continue;
            }
            // Exclusive key bound of this row (bottom-right causal alignment).
            int limit = u.L;
            if (p.causal) limit = imin(limit, qi + u.L - p.Sq + 1);
            limit = imax(limit, 0);
            float mneg = 0.f;  // -m_w (log2 units)
            int e = 0;         // m_w - m_O
            float qk_rowmax = -INFINITY;

            // Handshakes from the other warp of this quarter. The m_O handshake (once
            // per unit, early in its first tile) gives the reference of O; the
            // handshake of tile gi (at its end) gives the shift E applied to O before
            // P V(gi).
            auto receive_mo = [&]() -> bool {
                if (!__all_sync(0xffffffffu, wait_bar(&mo_bar[quarter], c & 1, abort_flag, p.status))) return false;
                const float m0 = __uint_as_float(lds32(a_m));
                mneg = m0 > -INFINITY ? -m0 : 0.f;
                e = 0;
                return true;
            };
            auto receive = [&](int gj) -> bool {
                if (!__all_sync(0xffffffffu, wait_bar(&hs[gj & 1], (gj >> 1) & 1, abort_flag, p.status)))
                    return false;
                e -= static_cast<int>(lds32(a_e + (gj & 1) * 128));
                return true;
            };

            for (int i = (pp - g) & 1; i < T; i += 2) {
                const int gi = g + i;  // global tile index: S buffer, P buffer and barrier parity gi & 1 == pp
                const int k = gi >> 1;
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
                        if (lane == 0) mbar_arrive(&s_free[pp]);  // the tensor core may now compute S(gi+2)
                    }
                    if (p.test_dump_s && blockIdx.x == 0 && c == 0 && i == 0) {
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
                        // The first half of the unit's first tile fixes m_O = m_w: the row's
                        // largest score there. It holds key 0, so a row with no key in it
                        // has none at all. The m_O handshake, posted now, gives it to the
                        // other warp.
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
                                const float2 uu = ffma2(make_float2(__uint_as_float(sh[j]), __uint_as_float(sh[j + 1])),
                                                        make_float2(sc, sc), make_float2(madd, madd));
                                const __half2 ph = __floats2half2_rn(exp2_approx(uu.x), exp2_approx(uu.y));
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
                    // P buffer pp was last read by P V(gi-2), issued at the end of this
                    // warp's previous tile.
                    if (hh == 0 && gi >= 2 &&
                        !__all_sync(0xffffffffu, wait_bar(&pv_done[pp], (k - 1) & 1, abort_flag, p.status))) {
                        ok = false;
                        break;
                    }
                    const uint32_t prow = smem_u32(pbuf) + row * 128;
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) {
                        const uint32_t cofs = static_cast<uint32_t>(((4 * hh + c2) ^ swz) << 4);
                        sts128(prow + cofs, pw[4 * c2], pw[4 * c2 + 1], pw[4 * c2 + 2], pw[4 * c2 + 3]);
                        sts128(prow + 128 * 128 + cofs, pw[16 + 4 * c2], pw[17 + 4 * c2], pw[18 + 4 * c2],
                               pw[19 + 4 * c2]);
                    }
                }
                if (!ok) break;
                if (kStageQK) continue;
                // Handshake with the other warp of this quarter, at the end of the tile:
                // take the shift E of tile gi-1 (it moved m_O), then decide this tile's.
                const int e_enc = e;
                if (i >= 1 && !receive(gi - 1)) {
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
                    // O holds P V up to tile gi-1 (the other warp's): wait for it, then
                    // scale this quarter's rows by 2^-E before P V(gi). (On a unit's first
                    // tile, P V(gi) overwrites O instead.)
                    if (!__all_sync(0xffffffffu,
                                    wait_bar(&pv_done[(gi - 1) & 1], ((gi - 1) >> 1) & 1, abort_flag, p.status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    rescale_o_lane(tmem + lane_base + kPfColO, 144, E);
                }
                // A warp that unwinds posts nothing; its peer's bounded wait then sees
                // the abort flag.
                sts32(a_e + (gi & 1) * 128, static_cast<uint32_t>(E));
                __syncwarp();
                if (lane == 0) mbar_arrive(&hs[gi & 1]);
                // Scale bytes of (row, block b): 2^(e + x) relative to m_O, with the
                // block's own e and the shifts of m_O since it was encoded. A block far
                // below m_O clamps at the smallest E8M0 value; it is negligible there.
                const int de_o = e - e_enc;
                uint32_t sfw = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    sfw |= static_cast<uint32_t>(imin(254, imax(0, 127 + eb[b] + de_o))) << (8 * b);
                sts32(smem_u32(smem + S::kSfP + pp * 512 + (row & 31) * 16 + (row >> 5) * 4), sfw);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[pp]);
            }
            if (!ok) break;
            // The warp that does not own the unit's last tile still applies its
            // handshake, so both warps of the quarter end with the same m_O = m_w - e.
            if (!kStageQK && ((g + T - 1) & 1) != pp) {
                if (T == 1) ok = receive_mo();  // this warp had no tile: take m_O first
                if (ok) ok = receive(g + T - 1);
                if (!ok) break;
            }
            // -------------------------------------------------------------- epilogue
            if (kStageQK) {
                // Each warp of the quarter posts its rows' maxima; the second to arrive
                // combines the two and writes them, so neither waits for the other.
                // A parity runs at most a few tiles (so units) ahead of the other,
                // well within the 8 slots.
                const int slot = c & 7;
                xmax[(slot * 2 + pp) * 128 + row] = qk_rowmax;
                __threadfence_block();
                __syncwarp();
                int second = 0;
                if (lane == 0) second = atomicAdd(&xcnt[quarter * 8 + slot], 1);
                second = __shfl_sync(0xffffffffu, second, 0);
                if (second) {
                    __threadfence_block();
                    const float m = fmaxf(xmax[(slot * 2) * 128 + row], xmax[(slot * 2 + 1) * 128 + row]);
                    if (row_valid && p.lse) p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] = m;
                    __syncwarp();
                    if (lane == 0) xcnt[quarter * 8 + slot] = 0;
                }
                g += T;
                ++c;
                continue;
            } else {
                ok = __all_sync(0xffffffffu, wait_bar(o_full, c & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                const float l = __uint_as_float(tc_ld_32x32b_x1(tmem + lane_base + kPfColO + 128));
                tc_wait_ld();
                // O and l are both relative to m_O = m_w - e.
                const bool anyk = l > 0.f;
                const float inv = anyk ? 1.f / l : 0.f;
                uint4 *dst = reinterpret_cast<uint4 *>(
                    p.out + ((static_cast<int64_t>(u.b) * p.Sq + qi) * p.Hq + u.h_q) * 128 + c_lo);
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
                                const int cc = 8 * q + 2 * kk;
                                const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(o[cc]) * inv,
                                                                                __uint_as_float(o[cc + 1]) * inv);
                                w[kk] = *reinterpret_cast<const uint32_t *>(&v2);
                            }
                            dst[4 * h + q] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                if (row_valid && pp == 0 && p.lse)
                    p.lse[(static_cast<int64_t>(u.b) * p.Hq + u.h_q) * p.Sq + qi] =
                        anyk ? (log2f(l) - mneg - static_cast<float>(e)) * 0.6931471805599453f : -INFINITY;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_free);  // the next unit's first P V may overwrite O
            }
            // Both warps of the quarter are done with this unit (its handshake slots).
            __syncwarp();
            if (lane == 0) mbar_arrive(&ue_bar[quarter]);
            ok = __all_sync(0xffffffffu, wait_bar(&ue_bar[quarter], c & 1, abort_flag, p.status));
            if (!ok) break;
            g += T;
            ++c;
        }
    }
    teardown_tmem(warp == kPfMmaWarp, tmem, kPfTmemCols);
}

template <bool kStageQK>
static cudaError_t launch_prefill_impl(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                       const AttnParams &p, cudaStream_t stream) {
    constexpr int kMaxDevices = 64;
    static bool configured[kMaxDevices] = {};
    static int sm_count[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int sms = dev < kMaxDevices ? sm_count[dev] : 0;
    if (dev >= kMaxDevices || !configured[dev]) {
        e = cudaFuncSetAttribute(qk4v8_prefill_kernel<kStageQK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 PfSmem::kBytes);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) {
            sm_count[dev] = sms;
            configured[dev] = true;
        }
    }
    // Persistent: one CTA per SM (shared memory and the 512 TMEM columns allow no
    // more), each walking the units blockIdx.x, blockIdx.x + grid, ...
    const int n_units = p.B * p.Hq * p.n_qtiles;
    const int grid = n_units < sms ? n_units : sms;
    qk4v8_prefill_kernel<kStageQK><<<grid, kPfThreads, PfSmem::kBytes, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p,
                           cudaStream_t stream) {
    return launch_prefill_impl<false>(tq, tk, tv, p, stream);
}

cudaError_t launch_prefill_stage_qk(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                    const AttnParams &p, cudaStream_t stream) {
    return launch_prefill_impl<true>(tq, tk, tv, p, stream);
}

}  // namespace qk4v8
