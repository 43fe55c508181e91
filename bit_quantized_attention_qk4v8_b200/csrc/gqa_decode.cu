// GQA decode / speculative-verify kernel for 33..64 query rows per KV head on
// sm_100a (MpFA QK4V8 article, sections 1.3, 2.1-2.3 and 3.3: decode attention
// streams the KV cache, 4-bit Q K^T, FP32 online softmax, 8-bit P V).
//
// The rows of one (sequence, KV head) are the G*nq query rows of its GQA group
// (row n = query head h_kv*G + n/nq at block token n%nq), at most 64. One CTA
// per SM walks the (sequence, KV head, key split) units. The softmax threads own
// one query row each, as in the prefill kernel, and all four TMEM lane quarters
// take part although the tile has only 64 rows:
//
//   - The Q buffer holds 192 rows [Q; 0; Q]. Rows 0..127 are Qa = [Q; 0] and
//     rows 64..191 are Qb = [0; Q], two K-major A operands that share one scale
//     atom (row n and row 64+n carry row n's scales).
//   - Key tiles go in pairs. S(pair) = Qa K(2k)^T, then += Qb K(2k+1)^T, into
//     one 128-column TMEM buffer: lanes 0..63 hold the scores of tile 2k and
//     lanes 64..127 those of tile 2k+1 (each MMA adds zero to the other half).
//   - P is stacked along M: the P tile of key tile t has P_hi of the 64 rows in
//     rows 0..63 and P_lo in rows 64..127, so O += P V is one set of four
//     kind::mxf8f6f4 MMAs (N = 144, V with a row of ones) per key tile. O lanes
//     0..63 accumulate the P_hi parts and lanes 64..127 the P_lo parts of both
//     tiles; column 128 is the matching part of the softmax denominator.
//
// Softmax warps 0..7: set = warp / 4 takes the pairs of its parity (S and P
// double-buffered by set); quarter q of the set reads TMEM lanes 32q..32q+31:
// quarters 0,1 the rows of tile 2k, quarters 2,3 the same rows for tile 2k+1.
// So four threads own each row: (set, tile half). Each keeps its own reference
// max m_w (moved by whole binades when a score passes it by 2^8), with an
// integer offset e = m_w - m_O to the row's common O reference m_O (the max of
// the first half of the unit's first tile). P = 2^(s*scale - m_w - x) per
// 32-key block, the block scale byte 127 + e + x. When an offset passes 2^64
// both threads of the set that own the row (whose O lanes are r and r+64)
// scale their lanes by the same 2^-E, agreed through a two-way exchange, and
// pass E on to the other set.
//
// Warp roles (384 threads): warps 0..7 softmax and epilogue, warp 8 TMA
// producer of K, warp 9 TMEM allocator and single-thread tcgen05 issuer,
// warp 10 TMA producer of V, warp 11 stages each unit's packed query rows. Splits write fp32 partials
// (O / l, log2-sum-exp) for the merge kernel; one split writes bf16 directly.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pipeline.cuh"
#include "ptx.cuh"
#include "qk4v8_internal.h"
#include "schedule.cuh"
#include "tile_ops.cuh"

namespace qk4v8 {

namespace {

constexpr int kGdKStages = 6;             // K tiles in flight (freed when the pair's QK^T completes)
constexpr int kGdVStages = 4;             // V tiles in flight (freed when the pair's P V completes)
constexpr int kGdSoftmaxWarps = 8;
constexpr int kGdThreads = 32 * kGdSoftmaxWarps + 128;
constexpr int kGdProducerWarp = 8;   // K
constexpr int kGdMmaWarp = 9;
constexpr int kGdVProducerWarp = 10;
constexpr int kGdQWarp = 11;
constexpr float kGdTau = 8.0f;             // m_w moves once a score passes it by 2^8
constexpr int kGdEMax = 64;                // largest offset e before O is rescaled
constexpr float kGdMaxMove = 16777216.0f;  // cap on one move of m_w, keeps it an exact integer

// Shared memory map (byte offsets from a 1024-aligned base).
struct GdSmem {
    static constexpr int kQRows = 192;                      // [Q; 0; Q]
    static constexpr int kQBytes = kQRows * 64;             // 64-byte swizzle
    static constexpr int kQ = 0;                            // 2 buffers (units alternate)
    static constexpr int kKBytes = 128 * 64;
    static constexpr int kK = kQ + 2 * kQBytes;             // per stage: 128 keys x 64 B
    static constexpr int kVRows = 144;                      // 128 channels, ones row, 15 zero rows
    static constexpr int kVBytes = kVRows * 128;
    static constexpr int kVTmaBytes = 128 * 128;
    static constexpr int kV = kK + kGdKStages * kKBytes;    // per stage: 144 rows x 128 B, 128-byte swizzle
    static constexpr int kPTile = 128 * 128;                // P_hi rows 0..63, P_lo rows 64..127
    static constexpr int kP = kV + kGdVStages * kVBytes;    // [set][tile half]
    static constexpr int kSfQ = kP + 4 * kPTile;            // 512-byte scale atoms: 2 Q buffers
    static constexpr int kSfK = kSfQ + 2 * 512;
    static constexpr int kSfV = kSfK + kGdKStages * 512;
    static constexpr int kSfP = kSfV + kGdVStages * 512;    // [set][tile half]
    static constexpr int kSfOne = kSfP + 4 * 512;
    static constexpr int kHsE = kSfOne + 512;               // int [pair parity][64 rows]: shift E of O
    static constexpr int kHsM = kHsE + 2 * 64 * 4;          // float [64 rows]: m_O of the unit
    static constexpr int kXe = kHsM + 64 * 4;               // int [set][tile half][parity][64 rows]
    static constexpr int kBar = kXe + 2 * 2 * 2 * 64 * 4;
    // k_full/k_empty, v_full/v_empty per stage; q_full/q_empty per Q buffer;
    // patch; s_full, s_free, p_full, pv_done per set; o_full, o_free, drain;
    // hs [pair parity][row group]; mo [row group]; ue [row group];
    // xb [set][row group][tile half][parity].
    static constexpr int kNumBars = 2 * kGdKStages + 2 * kGdVStages + 4 + 1 + 8 + 3 + 4 + 2 + 2 + 16;
    static constexpr int kMisc = kBar + kNumBars * 8;    // TMEM address, abort flag
    static constexpr int kSched = kMisc + 16;            // GdSched
    static constexpr int kUsed = kSched + 64;
    static constexpr int kBytes = kUsed + 1024;  // slack for aligning the base
};
static_assert(GdSmem::kQBytes % 1024 == 0 && GdSmem::kK % 1024 == 0 && GdSmem::kV % 1024 == 0 &&
                  GdSmem::kP % 1024 == 0 && GdSmem::kVBytes % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
static_assert(GdSmem::kBar % 8 == 0, "mbarrier alignment");
static_assert(GdSmem::kBytes <= 227 * 1024, "shared memory budget");

// TMEM columns (512 allocated, one CTA per SM).
constexpr uint32_t kGdTmemCols = 512;
constexpr uint32_t kGdColO = 256;  // 144 columns: O[:, 0:128], the denominator part in column 128
__device__ __forceinline__ uint32_t gd_col_s(int set) { return 128u * set; }
__device__ __forceinline__ uint32_t gd_col_sf_q(int qb) { return 400u + 4u * qb; }
__device__ __forceinline__ uint32_t gd_col_sf_k(int set, int h) { return 408u + 8u * set + 4u * h; }
// V scales per (set, tile half): 4 columns, then 4 constant columns for the ones row.
__device__ __forceinline__ uint32_t gd_col_sf_v(int set, int h) { return 424u + 16u * set + 8u * h; }
__device__ __forceinline__ uint32_t gd_col_sf_p(int set, int h) { return 456u + 8u * set + 4u * h; }

constexpr uint32_t gd_idesc(uint32_t fmt, uint32_t n) {
    return (fmt << 7) | (fmt << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}
constexpr uint32_t kGdIdQK = gd_idesc(1u, 128);             // E2M1 x E2M1, N = 128 keys
constexpr uint32_t kGdIdPV = gd_idesc(0u, GdSmem::kVRows);  // E4M3 x E4M3, N = 144
__device__ __forceinline__ uint32_t gd_sf_id(uint32_t idesc, uint32_t id) { return idesc | (id << 29) | (id << 4); }

}  // namespace

// kExt: the instance for draft-block attention (query rows see only keys from
// the window's first key, kv_window_lo, on), paged caches (key tiles looked up
// in the block table) and MXFP4 V (the QK4V4 comparison point); the other
// instance is the plain decode over a contiguous MXFP8-V cache, with none of
// these in its loops.
template <bool kExt>
__global__ void __launch_bounds__(kGdThreads, 1)
    qk4v8_gqa_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                            const AttnParams p) {
    using S = GdSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nq = p.Sq;
    const int R = p.G * nq;  // query rows of a unit, 33..64

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::kBar);
    uint64_t *k_full = bars;
    uint64_t *k_empty = k_full + kGdKStages;
    uint64_t *v_full = k_empty + kGdKStages;
    uint64_t *v_empty = v_full + kGdVStages;
    uint64_t *q_full = v_empty + kGdVStages;  // [Q buffer]
    uint64_t *q_empty = q_full + 2;           // [Q buffer]
    uint64_t *patch = q_empty + 2;
    uint64_t *s_full = patch + 1;    // [set]
    uint64_t *s_free = s_full + 2;   // [set]
    uint64_t *p_full = s_free + 2;   // [set]
    uint64_t *pv_done = p_full + 2;  // [set]
    uint64_t *o_full = pv_done + 2;
    uint64_t *o_free = o_full + 1;
    uint64_t *drain = o_free + 1;
    uint64_t *hs_bar = drain + 1;   // [pair parity][row group]
    uint64_t *mo_bar = hs_bar + 4;  // [row group]
    uint64_t *ue_bar = mo_bar + 2;  // [row group]: the four warps of the rows are done with a unit
    uint64_t *xb_bar = ue_bar + 2;  // [set][row group][tile half][parity]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMisc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + S::kMisc + 4);
    GdSched *sched = reinterpret_cast<GdSched *>(smem + S::kSched);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGdKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kGdVStages; ++s) {
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
        mbar_init(o_free, kGdSoftmaxWarps);
        mbar_init(drain, 1);
        for (int g = 0; g < 4; ++g) mbar_init(&hs_bar[g], 1);
        for (int g = 0; g < 2; ++g) {
            mbar_init(&mo_bar[g], 1);
            mbar_init(&ue_bar[g], 4);
        }
        for (int g = 0; g < 16; ++g) mbar_init(&xb_bar[g], 1);
        // A status already set by another launch or CTA: unwind at once (every
        // wait returns false), uniformly for the whole CTA.
        *abort_flag = (p.status && *reinterpret_cast<const volatile int32_t *>(p.status) != 0) ? 1u : 0u;
        fence_barrier_init();
    }
    if (warp == kGdMmaWarp) {
        tmem_alloc(tmem_slot, kGdTmemCols);
        tmem_relinquish();
    }
    if (warp == 0) gd_schedule(p, *sched);
    // Both Q buffers and their scale atoms start at zero: rows R..63 and 64..127
    // (and 128+R..191) are never written again, and zero codes with zero
    // scales contribute nothing.
    for (int i = threadIdx.x; i < 2 * S::kQBytes / 16; i += kGdThreads)
        reinterpret_cast<uint4 *>(smem + S::kQ)[i] = make_uint4(0, 0, 0, 0);
    for (int i = threadIdx.x; i < 2 * 512 / 16; i += kGdThreads)
        reinterpret_cast<uint4 *>(smem + S::kSfQ)[i] = make_uint4(0, 0, 0, 0);
    if (warp == kGdVProducerWarp) {
        // Constant V rows: row 128 = 1.0 (E4M3 0x38), rows 129..143 = 0, and a
        // scale atom of 2^0 for them. TMA never writes these rows.
        for (int s = 0; s < kGdVStages; ++s)
            for (int cc = lane; cc < 16 * 8; cc += 32) {
                const int r = 128 + (cc >> 3);
                // 1.0 is E4M3 0x38; with MXFP4 V (extended instance) it is E2M1 0x2,
                // and 0x22 in every byte gives two 1.0 codes whichever 8 bytes of each
                // 16-byte slot the padded FP4 layout reads.
                const uint32_t one = kExt && p.v_fp4 ? 0x22222222u : 0x38383838u;
                const uint32_t fillv = r == 128 ? one : 0u;
                *reinterpret_cast<uint4 *>(smem + S::kV + s * S::kVBytes + r * 128 + (cc & 7) * 16) =
                    make_uint4(fillv, fillv, fillv, fillv);
            }
        reinterpret_cast<uint4 *>(smem + S::kSfOne)[lane] = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const GdSched gs = *sched;

    if (warp == kGdProducerWarp) {
        // ------------------------------------------------------------- K producer
        if (lane == 0) prefetch_tensormap(&tmap_k);
        const int nblk = kv_row_blocks<kExt>(p);
        PageLookup pl;
        int g = 0;  // tiles so far
        int gk_issued = 0;
        bool ok = true;
        GdIter it;
        gd_begin(p, gs, it);
        GdUnit u;
        while (ok && gd_next(p, gs, it, u)) {
            const int T = u.T;
            if (T <= 0) continue;
            // K tiles of the unit: the K ring frees as soon as the pair's QK^T
            // completes, so K runs up to kGdKStages tiles ahead of the tensor core.
            for (int it = 0; it < T && ok; ++it) {
                const int gk = g + it;
                const int st = gk % kGdKStages;
                ok = __all_sync(0xffffffffu, wait_bar(&k_empty[st], ((gk / kGdKStages) & 1) ^ 1, abort_flag, p.status));
                if (!ok) break;
                int row, blk;
                kv_tile_row<kExt>(p, u.b, u.h_kv, u.tile_begin + it, pl, row, blk);
                if (lane == 0) {
                    mbar_arrive_expect_tx(&k_full[st], S::kKBytes + 512);
                    tma_load_3d(smem + S::kK + st * S::kKBytes, &tmap_k, 0, blk * 128, row, &k_full[st]);
                    bulk_load(smem + S::kSfK + st * 512, p.k_scales + (static_cast<int64_t>(row) * nblk + blk) * 512,
                              512, &k_full[st]);
                }
                gk_issued = gk + 1;
            }
            g += T;
        }
        // Let every issued copy land before the CTA can retire.
        if (lane == 0) {
            for (int gk = imax(0, gk_issued - kGdKStages); gk < gk_issued; ++gk) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&k_full[gk % kGdKStages], (gk / kGdKStages) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
        }
    } else if (warp == kGdQWarp) {
        // ------------------------------------------------------------ Q staging
        // The packed query rows of each unit into Q buffer c & 1, while earlier
        // units run: codes to rows n and 128 + n (64-byte swizzle: chunk j of
        // row n at j ^ ((n / 2) % 4)), the row's scale word to atom rows n and
        // 64 + n. The MMA warp frees the buffer after the unit's last QK^T.
        int c = 0;  // units staged
        bool ok = true;
        auto stage_q = [&](const GdUnit &v) -> bool {
            const int qb = c & 1;
            if (!__all_sync(0xffffffffu, wait_bar(&q_empty[qb], ((c >> 1) & 1) ^ 1, abort_flag, p.status)))
                return false;
            uint8_t *qbuf = smem + S::kQ + qb * S::kQBytes;
            uint8_t *sfq = smem + S::kSfQ + qb * 512;
            uint4 qv[8];
            uint32_t sv[2];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int idx = lane + 32 * i, n = idx >> 2, jj = idx & 3;
                qv[i] = make_uint4(0, 0, 0, 0);
                if (n < R) {
                    const int h = v.h_kv * p.G + n / nq, t = n % nq;
                    qv[i] = *reinterpret_cast<const uint4 *>(
                        p.q_codes + ((static_cast<int64_t>(v.b) * p.Hq + h) * p.q_cap + t) * 64 + jj * 16);
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int n = lane + 32 * i;
                sv[i] = 0;
                if (n < R) {
                    const int h = v.h_kv * p.G + n / nq, t = n % nq;
                    sv[i] = *reinterpret_cast<const uint32_t *>(
                        p.q_scales + ((static_cast<int64_t>(v.b) * p.Hq + h) * (p.q_cap / 128) + t / 128) * 512 +
                        (t & 31) * 16 + ((t & 127) >> 5) * 4);
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int idx = lane + 32 * i, n = idx >> 2, jj = idx & 3;
                if (n < R) {
                    const int cofs = (jj ^ ((n >> 1) & 3)) << 4;
                    *reinterpret_cast<uint4 *>(qbuf + n * 64 + cofs) = qv[i];
                    *reinterpret_cast<uint4 *>(qbuf + (128 + n) * 64 + cofs) = qv[i];
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int n = lane + 32 * i;
                if (n < R) {
                    *reinterpret_cast<uint32_t *>(sfq + (n & 31) * 16 + (n >> 5) * 4) = sv[i];
                    *reinterpret_cast<uint32_t *>(sfq + (n & 31) * 16 + ((n >> 5) + 2) * 4) = sv[i];
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && !(p.test_stall && c == 0)) mbar_arrive(&q_full[qb]);
            ++c;
            return true;
        };
        GdIter it;
        gd_begin(p, gs, it);
        GdUnit u;
        while (ok && gd_next(p, gs, it, u))
            if (u.T > 0) ok = stage_q(u);
    } else if (warp == kGdVProducerWarp) {
        // -------------------------------------------------------------- V producer
        // V tiles on their own warp, so that a V stage waiting for its P V never
        // holds back the K loads of later pairs.
        if (lane == 0) prefetch_tensormap(&tmap_v);
        const int nblk = kv_row_blocks<kExt>(p);
        PageLookup pl;
        int g = 0, gv_issued = 0;
        bool ok = true;
        GdIter it;
        gd_begin(p, gs, it);
        GdUnit u;
        while (ok && gd_next(p, gs, it, u)) {
            const int T = u.T;
            if (T <= 0) continue;
            const bool last_partial = (u.L & 127) != 0 && u.tile_begin + T == (u.L + 127) / 128;
            for (int jt = 0; jt < T && ok; ++jt) {
                const int gv = g + jt;
                const int sv = gv % kGdVStages;
                const uint32_t ph = (gv / kGdVStages) & 1;
                ok = __all_sync(0xffffffffu, wait_bar(&v_empty[sv], ph ^ 1, abort_flag, p.status));
                if (!ok) break;
                const int tile = u.tile_begin + jt;
                int row, blk;
                kv_tile_row<kExt>(p, u.b, u.h_kv, tile, pl, row, blk);
                if (lane == 0) {
                    // An MXFP4 tile lands unpacked; the copy moves half the bytes.
                    mbar_arrive_expect_tx(&v_full[sv], (kExt && p.v_fp4 ? S::kVTmaBytes / 2 : S::kVTmaBytes) + 512);
                    tma_load_3d(smem + S::kV + sv * S::kVBytes, &tmap_v, 0, 0, row * nblk + blk, &v_full[sv]);
                    bulk_load(smem + S::kSfV + sv * 512, p.v_scales + (static_cast<int64_t>(row) * nblk + blk) * 512,
                              512, &v_full[sv]);
                }
                gv_issued = gv + 1;
                if (last_partial && jt == T - 1) {
                    // Keys at or past L may hold anything (a reused cache). Their P is
                    // zero, but a NaN code or scale in V would still poison O: zero them
                    // once the tile has landed, and tell the MMA warp.
                    ok = __all_sync(0xffffffffu, wait_bar(&v_full[sv], ph, abort_flag, p.status));
                    if (!ok) break;
                    const int jv = u.L - tile * 128;  // valid keys in this tile, 1..127
                    uint8_t *vt = smem + S::kV + sv * S::kVBytes;
                    // (E2M1 has no NaN or infinity: MXFP4 V codes need no zeroing.)
                    for (int cc = lane; cc < 128 * 8 && !(kExt && p.v_fp4); cc += 32) {
                        const int r = cc >> 3, q = cc & 7;
                        if (16 * q + 16 <= jv) continue;
                        uint8_t *chunk = vt + r * 128 + ((q ^ (r & 7)) << 4);
                        for (int e = 0; e < 16; ++e)
                            if (16 * q + e >= jv) chunk[e] = 0;
                    }
                    uint8_t *sfv = smem + S::kSfV + sv * 512;
                    for (int r = lane; r < 128; r += 32)
                        for (int gq = (jv + 31) / 32; gq < 4; ++gq) sfv[(r & 31) * 16 + (r >> 5) * 4 + gq] = 0;
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(patch);
                }
            }
            g += T;
        }
        if (lane == 0) {
            for (int gv = imax(0, gv_issued - kGdVStages); gv < gv_issued; ++gv) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&v_full[gv % kGdVStages], (gv / kGdVStages) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
        }
    } else if (warp == kGdMmaWarp) {
        // -------------------------------------------------------------- MMA issuer
        // The whole warp runs the loop and waits, so the descriptors stay
        // warp-uniform; one elected lane issues the tcgen05 instructions.
        uint32_t pred;
        asm volatile(
            "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.u32 %0, 1, 0, e;\n\t}"
            : "=r"(pred));
        const bool leader = pred != 0;
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
        const uint32_t tO = tmem + kGdColO;
        // The ones row's scale, for all four V scale slots, once.
        if (leader) {
            const uint64_t dOne = smem_desc(sb + S::kSfOne, 0, 128, 0);
            for (int s = 0; s < 2; ++s)
                for (int h = 0; h < 2; ++h) tc_cp_32x128b_warpx4(tmem + gd_col_sf_v(s, h) + 4, dOne);
        }
        __syncwarp();
        bool ok = true;
        int g = 0, gp0 = 0, c = 0, n_patch = 0;  // tiles, pairs and units so far
        GdIter it;
        gd_begin(p, gs, it);
        GdUnit u;
        while (ok && gd_next(p, gs, it, u)) {
            const int T = u.T;
            if (T <= 0) continue;
            const int NP = (T + 1) / 2;
            const int qb = c & 1;
            const bool last_partial = (u.L & 127) != 0 && u.tile_begin + T == (u.L + 127) / 128;
            ok = __all_sync(0xffffffffu, wait_bar(&q_full[qb], (c >> 1) & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tSfQ = tmem + gd_col_sf_q(qb);
            const uint64_t dQa = dQ0 + static_cast<uint64_t>(qb * (S::kQBytes >> 4));
            const uint64_t dQb = dQa + static_cast<uint64_t>((64 * 64) >> 4);  // rows 64..191
            if (leader) tc_cp_32x128b_warpx4(tSfQ, dSfQ0 + static_cast<uint64_t>(qb * 32));
            __syncwarp();
            // S(pair k) = Qa K(2k)^T + Qb K(2k+1)^T into the S buffer of set gp & 1,
            // once both K tiles have landed and the set has read S(gp - 2).
            auto issue_qk = [&](int k) -> bool {
                const int gp = gp0 + k, set = gp & 1;
                const bool has1 = 2 * k + 1 < T;
                const int gk0 = g + 2 * k, gk1 = gk0 + 1;
                const int st0 = gk0 % kGdKStages, st1 = gk1 % kGdKStages;
                bool w = wait_bar(&k_full[st0], (gk0 / kGdKStages) & 1, abort_flag, p.status);
                if (w && has1) w = wait_bar(&k_full[st1], (gk1 / kGdKStages) & 1, abort_flag, p.status);
                if (w && gp >= 2) w = wait_bar(&s_free[set], ((gp - 2) >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, w)) return false;
                tc_fence_after();
                const uint32_t tS = tmem + gd_col_s(set);
                const uint32_t tSfK0 = tmem + gd_col_sf_k(set, 0), tSfK1 = tmem + gd_col_sf_k(set, 1);
                const uint64_t dK0s = dK0 + static_cast<uint64_t>(st0 * (S::kKBytes >> 4));
                const uint64_t dK1s = dK0 + static_cast<uint64_t>(st1 * (S::kKBytes >> 4));
                if (leader) {
                    tc_cp_32x128b_warpx4(tSfK0, dSfK0 + static_cast<uint64_t>(st0 * 32));
                    if (has1) tc_cp_32x128b_warpx4(tSfK1, dSfK0 + static_cast<uint64_t>(st1 * 32));
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc_mma_mxf4(tS, dQa + 2 * kk, dK0s + 2 * kk, gd_sf_id(kGdIdQK, 2 * kk), tSfQ | ((2u * kk) << 30),
                                    tSfK0 | ((2u * kk) << 30), kk > 0 ? 1u : 0u);
                    if (has1) {
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk)
                            tc_mma_mxf4(tS, dQb + 2 * kk, dK1s + 2 * kk, gd_sf_id(kGdIdQK, 2 * kk),
                                        tSfQ | ((2u * kk) << 30), tSfK1 | ((2u * kk) << 30), 1u);
                    }
                    tc_commit(&s_full[set]);
                    tc_commit(&k_empty[st0]);
                    if (has1) tc_commit(&k_empty[st1]);
                }
                __syncwarp();
                return true;
            };
            // O += P(2k) V(2k) + P(2k+1) V(2k+1), once both V tiles have landed and
            // the set has written its P tiles; the unit's first one overwrites O,
            // once the previous unit's epilogue has read it.
            // E4M3 P x E4M3 V, N = 144; with MXFP4 V the B format field says E2M1 (5).
            const uint32_t id_pv = kGdIdPV | (kExt && p.v_fp4 ? (5u << 10) : 0u);
            auto issue_pv = [&](int k) -> bool {
                const int gp = gp0 + k, set = gp & 1;
                const bool has1 = 2 * k + 1 < T;
                const int gv0 = g + 2 * k, gv1 = gv0 + 1;
                const int sv0 = gv0 % kGdVStages, sv1 = gv1 % kGdVStages;
                bool w = wait_bar(&v_full[sv0], (gv0 / kGdVStages) & 1, abort_flag, p.status);
                if (w && has1) w = wait_bar(&v_full[sv1], (gv1 / kGdVStages) & 1, abort_flag, p.status);
                if (w && last_partial && (2 * k == T - 1 || 2 * k + 1 == T - 1))
                    w = wait_bar(patch, n_patch & 1, abort_flag, p.status);
                if (w && k == 0 && c >= 1) w = wait_bar(o_free, (c - 1) & 1, abort_flag, p.status);
                if (w) w = wait_bar(&p_full[set], (gp >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, w)) return false;
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h == 1 && !has1) break;
                        const int sv = h ? sv1 : sv0;
                        const uint32_t tSfV = tmem + gd_col_sf_v(set, h);
                        const uint32_t tSfP = tmem + gd_col_sf_p(set, h);
                        const uint64_t dV = dV0 + static_cast<uint64_t>(sv * (S::kVBytes >> 4));
                        const uint64_t dP = dP0 + static_cast<uint64_t>((2 * set + h) * (S::kPTile >> 4));
                        tc_cp_32x128b_warpx4(tSfV, dSfV0 + static_cast<uint64_t>(sv * 32));
                        tc_cp_32x128b_warpx4(tSfP, dSfP0 + static_cast<uint64_t>((2 * set + h) * 32));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma_mxf8(tO, dP + 2 * kk, dV + 2 * kk, gd_sf_id(id_pv, kk), tSfP | (kk << 30),
                                        tSfV | (kk << 30), (k > 0 || h > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(&pv_done[set]);
                    tc_commit(&v_empty[sv0]);
                    if (has1) tc_commit(&v_empty[sv1]);
                }
                __syncwarp();
                return true;
            };
            // The tensor pipe runs in issue order, so the issue order follows the order
            // in which the softmax sets release their inputs: S(k) is read early in
            // pair k, P(k-1) is written at the end of pair k-1 by the other set. So:
            // S(0), S(1), then per pair k: S(k+2) once S(k) has been read, then
            // P(k-1) V(k-1).
            ok = issue_qk(0);
            if (ok && NP > 1) ok = issue_qk(1);
            for (int k = 0; k < NP && ok; ++k) {
                if (k + 2 < NP) ok = issue_qk(k + 2);
                if (ok && k >= 1) ok = issue_pv(k - 1);
            }
            if (ok) ok = issue_pv(NP - 1);
            if (!ok) break;
            if (leader) {
                tc_commit(&q_empty[qb]);  // Q buffer and its scale columns free for unit c + 2
                tc_commit(o_full);
            }
            __syncwarp();
            if (last_partial) ++n_patch;
            g += T;
            gp0 += NP;
            ++c;
        }
        // Every tcgen05 operation issued above has completed once `drain` does, also
        // when the loop unwound early, so TMEM is freed with nothing in flight.
        if (leader) tc_commit(drain);
        __syncwarp();
        (void)wait_peers(drain, 0);
    } else if (warp < kGdSoftmaxWarps) {
        // ------------------------------------------------------------------ softmax
        const int set = warp >> 2;      // owns the pairs whose global index has this parity
        const int quarter = warp & 3;   // TMEM lane quarter this warp may access
        const int grp = quarter & 1;    // row group: rows 32 grp .. 32 grp + 31
        const int half = quarter >> 1;  // 0: the pair's first tile (lanes 0..63); 1: its second (64..127)
        const int r = 32 * grp + lane;  // query row of the unit
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int swz = r & 7;
        const uint32_t p_base = smem_u32(smem + S::kP);
        const uint32_t p_hi = p_base + (2 * set + half) * S::kPTile + r * 128;  // P_hi row r; P_lo row r + 64
        const uint32_t a_sf = smem_u32(smem + S::kSfP) + (2 * set + half) * 512 + (r & 31) * 16 + (r >> 5) * 4;
        const uint32_t a_e = smem_u32(smem + S::kHsE) + r * 4;  // + pair parity * 256
        const uint32_t a_m = smem_u32(smem + S::kHsM) + r * 4;
        const uint32_t a_x = smem_u32(smem + S::kXe) + (set * 2 + half) * 512 + r * 4;       // + parity * 256
        const uint32_t a_xo = smem_u32(smem + S::kXe) + (set * 2 + 1 - half) * 512 + r * 4;  // partner's slot
        uint64_t *xb_mine = xb_bar + ((set * 2 + grp) * 2 + half) * 2;       // [parity]
        uint64_t *xb_other = xb_bar + ((set * 2 + grp) * 2 + 1 - half) * 2;  // [parity]
        const float sc = p.scale_log2;
        const bool row_valid = r < R;
        const int c_lo = 64 * set + 32 * half;        // output columns this thread finalizes
        const int c_send = 64 * set + 32 * (1 - half);  // columns it hands to the partner
        int gpair = 0, c = 0, nx = 0;  // pairs and units so far; exchanges with the partner
        bool ok = true;
        // Two-way exchange with the other thread of this set that owns row r (the
        // other tile half): post this thread's arrival, wait for the partner's.
        auto meet = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&xb_mine[nx & 1]);
            const bool w = __all_sync(0xffffffffu, wait_bar(&xb_other[nx & 1], (nx >> 1) & 1, abort_flag, p.status));
            ++nx;
            return w;
        };
        // Final bf16 columns c_lo .. c_lo+31 of row r (and, for one thread of the
        // row, its natural-log lse) from O / l and the log2-sum-exp.
        auto write_out = [&](const GdUnit &v, const float (&o)[32], float lse2) {
            const int h_q = v.h_kv * p.G + r / nq, tq = r % nq;
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((static_cast<int64_t>(v.b) * nq + tq) * p.Hq + h_q) * 128 +
                                                   c_lo);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t w[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const __nv_bfloat162 v2 = __floats2bfloat162_rn(o[8 * q + 2 * kk], o[8 * q + 2 * kk + 1]);
                    w[kk] = *reinterpret_cast<const uint32_t *>(&v2);
                }
                dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (c_lo == 0 && p.lse)
                p.lse[(static_cast<int64_t>(v.b) * p.Hq + h_q) * nq + tq] =
                    lse2 > -INFINITY ? lse2 * 0.6931471805599453f : -INFINITY;
        };
        // Finishes unit v for this thread's columns: in the direct-output call a
        // whole sequence goes straight to the output; otherwise the piece is
        // written as the fp32 partial of its slot, for the merge kernel.
        auto finish = [&](const GdUnit &v, const float (&o)[32], float lse2) {
            // The merge launch reads, per sequence, how many pieces to merge: 0 when
            // the sequence was written whole. The piece in slot 0 records it.
            if (p.direct_out && p.piece_counts && v.slot == 0 && warp == 0 && lane == 0)
                p.piece_counts[v.b * p.Hkv + v.h_kv] = v.whole ? 0 : v.n_pieces;
            if (!row_valid) return;
            if (v.whole && p.direct_out) {
                write_out(v, o, lse2);
                return;
            }
            const int h_q = v.h_kv * p.G + r / nq, tq = r % nq;
            const int64_t prow = ((static_cast<int64_t>(v.b) * p.Hq + h_q) * nq + tq) * p.num_splits + v.slot;
            float4 *dst = reinterpret_cast<float4 *>(p.ws_o + prow * 128 + c_lo);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            if (c_lo == 0) p.ws_lse[prow] = lse2;
        };
        GdIter it;
        gd_begin(p, gs, it);
        GdUnit u;
        while (ok && gd_next(p, gs, it, u)) {
            const int T = u.T;
            const int tq = r % nq;
            if (T <= 0) {
                // A piece with no key: O = 0 and lse = -inf for every query row.
                float zero[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) zero[k] = 0.f;
                finish(u, zero, -INFINITY);
                continue;
            }
            // Exclusive key bound of this row (bottom-right causal alignment of the
            // nq-token block).
            int limit = u.L;
            if (p.causal) limit = imin(limit, u.L - nq + tq + 1);
            limit = imax(limit, 0);
            const int NP = (T + 1) / 2;
            float mneg = 0.f;  // -m_w (log2 units)
            int e = 0;         // m_w - m_O
            // m_O comes from the first half (64 keys) of the unit's first tile that
            // holds a visible key: the second half when a window starts there.
            const int u_lo = kExt ? kv_window_lo(p, u.L) : 0;  // the unit's first visible key
            const int mo_half = kExt && u_lo - u.tile_begin * 128 >= 64 ? 1 : 0;
            auto receive_mo = [&]() -> bool {
                if (!__all_sync(0xffffffffu, wait_bar(&mo_bar[grp], c & 1, abort_flag, p.status))) return false;
                const float m0 = __uint_as_float(lds32(a_m));
                mneg = m0 > -INFINITY ? -m0 : 0.f;
                e = 0;
                return true;
            };
            auto receive = [&](int gj) -> bool {
                if (!__all_sync(0xffffffffu,
                                wait_bar(&hs_bar[(gj & 1) * 2 + grp], (gj >> 1) & 1, abort_flag, p.status)))
                    return false;
                e -= static_cast<int>(lds32(a_e + (gj & 1) * 256));
                return true;
            };

            for (int k = (set - gpair) & 1; k < NP; k += 2) {
                const int gp = gpair + k;  // global pair index: S buffer, P tiles and barrier parity gp & 1 == set
                const int ti = 2 * k + half;  // this thread's key tile in the unit
                ok = __all_sync(0xffffffffu, wait_bar(&s_full[set], (gp >> 1) & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                const int jv = ti < T ? imax(0, imin(limit - (u.tile_begin + ti) * 128, 128)) : 0;  // keys j < jv
                const int jlo = kExt ? u_lo - (u.tile_begin + ti) * 128 : 0;  // and keys j >= jlo (window)
                int eb[4];  // e + x of each block when it was encoded
                // The tile in two halves of 64 keys, to bound the registers held at once.
                // S is released to the tensor core once the second half has been read.
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t sh[64];
                    uint32_t pw[32];  // this half's P bytes: P_hi words [0, 16), P_lo words [16, 32)
                    tc_ld_32x32b_x32(tmem + lane_base + gd_col_s(set) + 64 * hh,
                                     *reinterpret_cast<uint32_t (*)[32]>(&sh[0]));
                    tc_ld_32x32b_x32(tmem + lane_base + gd_col_s(set) + 64 * hh + 32,
                                     *reinterpret_cast<uint32_t (*)[32]>(&sh[32]));
                    tc_wait_ld();
                    if (hh == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&s_free[set]);  // the tensor core may now compute S(gp+2)
                    }
                    // Keys at or past the row's bound, and before the window, are -inf
                    // (raw scores; the scale is positive).
                    if (kExt) {
                        if (jv < 64 * hh + 64 || jlo > 64 * hh) {
#pragma unroll
                            for (int j = 0; j < 64; ++j)
                                if (64 * hh + j >= jv || 64 * hh + j < jlo) sh[j] = 0xFF800000u;
                        }
                    } else if (jv < 64 * hh + 64) {
#pragma unroll
                        for (int j = 0; j < 64; ++j)
                            if (64 * hh + j >= jv) sh[j] = 0xFF800000u;
                    }
                    const float bmx0 = max32(*reinterpret_cast<const uint32_t (*)[32]>(&sh[0])) * sc;
                    const float bmx1 = max32(*reinterpret_cast<const uint32_t (*)[32]>(&sh[32])) * sc;
                    const float hm = fmaxf(bmx0, bmx1);
                    const bool mo_post = k == 0 && half == 0 && hh == mo_half;
                    const bool mo_take = k == 0 && half == 1 && hh == 0;
                    if (kExt ? (mo_post || mo_take) : (k == 0 && hh == 0)) {
                        // The first half of the unit's first tile with a visible key fixes
                        // m_O: the row's largest score there. It holds the unit's first
                        // visible key, so a row with no key in it has none in the unit. Its
                        // owner posts it to the other three. (With a window, a half before
                        // it is all masked: its P is zero, whatever the reference.)
                        if (half == 0) {
                            mneg = hm > -INFINITY ? -hm : 0.f;
                            e = 0;
                            sts32(a_m, __float_as_uint(-mneg));
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&mo_bar[grp]);
                        } else if (!receive_mo()) {
                            ok = false;
                            break;
                        }
                    } else if (k == 1 && hh == 0 && !receive_mo()) {
                        ok = false;
                        break;
                    }
                    {
                        // m_w moves to the next whole binade above the half's max, so e
                        // stays integral.
                        const float bt = hm + mneg;
                        if (bt > kGdTau) {
                            const float de = ceilf(fminf(bt, kGdMaxMove));
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
                            for (int hf = 0; hf < 2; ++hf) {
                                const int j = 32 * b2 + 4 * q + 2 * hf;
                                const float2 uu = ffma2(make_float2(__uint_as_float(sh[j]), __uint_as_float(sh[j + 1])),
                                                        make_float2(sc, sc), make_float2(madd, madd));
                                const __half2 ph = __floats2half2_rn(exp2_approx(uu.x), exp2_approx(uu.y));
                                const uint32_t phw = *reinterpret_cast<const uint32_t *>(&ph);
                                const uint16_t h2 = cvt_e4m3x2_from_f16x2(phw);
                                const uint32_t hvw = cvt_e4m3x2_to_f16x2(h2);
                                const __half2 d = __hsub2(ph, *reinterpret_cast<const __half2 *>(&hvw));
                                hh2[hf] = h2;
                                ll2[hf] = cvt_e4m3x2_from_f16x2(*reinterpret_cast<const uint32_t *>(&d));
                            }
                            pw[8 * b2 + q] = __byte_perm(hh2[0], hh2[1], 0x5410);
                            pw[16 + 8 * b2 + q] = __byte_perm(ll2[0], ll2[1], 0x5410);
                        }
                    }
                    // The set's P tiles were last read by P V(gp-2), issued at the end of
                    // the set's previous pair.
                    if (hh == 0 && gp >= 2 &&
                        !__all_sync(0xffffffffu, wait_bar(&pv_done[set], ((gp >> 1) - 1) & 1, abort_flag, p.status))) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) {
                        const uint32_t cofs = static_cast<uint32_t>(((4 * hh + c2) ^ swz) << 4);
                        sts128(p_hi + cofs, pw[4 * c2], pw[4 * c2 + 1], pw[4 * c2 + 2], pw[4 * c2 + 3]);
                        sts128(p_hi + 64 * 128 + cofs, pw[16 + 4 * c2], pw[17 + 4 * c2], pw[18 + 4 * c2],
                               pw[19 + 4 * c2]);
                    }
                }
                if (!ok) break;
                // End of the pair: take the shift E of pair gp-1 (from the other set),
                // then agree with the partner (same row, other tile half) on this pair's
                // shift: both own half of the row's O (lanes r and r + 64).
                const int e_enc = e;
                if (k >= 1 && !receive(gp - 1)) {
                    ok = false;
                    break;
                }
                const int xp = nx & 1;
                sts32(a_x + xp * 256, static_cast<uint32_t>(e));
                if (!meet()) {
                    ok = false;
                    break;
                }
                const int em = imax(e, static_cast<int>(lds32(a_xo + xp * 256)));
                const int E = em > kGdEMax ? em : 0;
                e -= E;
                if (__any_sync(0xffffffffu, E != 0) && k >= 1) {
                    // O holds P V up to pair gp-1 (the other set's): wait for it, then
                    // scale this thread's lane of O by 2^-E before P V(gp). (On a unit's
                    // first pair, P V(gp) overwrites O instead.)
                    if (!__all_sync(0xffffffffu,
                                    wait_bar(&pv_done[set ^ 1], ((gp - 1) >> 1) & 1, abort_flag, p.status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    rescale_o_lane(tmem + lane_base + kGdColO, 144, E);
                }
                // A warp that unwinds posts nothing; the waiters' bounded waits then see
                // the abort flag.
                if (half == 0) {
                    sts32(a_e + (gp & 1) * 256, static_cast<uint32_t>(E));
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&hs_bar[(gp & 1) * 2 + grp]);
                }
                // Scale bytes of (row, block b), for the P_hi row r and the P_lo row
                // r + 64: 2^(e + x) relative to m_O, with the block's own e and the
                // shifts of m_O since it was encoded. A block far below m_O clamps at
                // the smallest E8M0 value; it is negligible there.
                const int de_o = e - e_enc;
                uint32_t sfw = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    sfw |= static_cast<uint32_t>(imin(254, imax(0, 127 + eb[b] + de_o))) << (8 * b);
                sts32(a_sf, sfw);
                sts32(a_sf + 8, sfw);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[set]);
            }
            if (!ok) break;
            // The set that does not own the unit's last pair still applies its
            // handshake, so all four owners of the row end with the same m_O = m_w - e.
            if (((gpair + NP - 1) & 1) != set) {
                if (NP == 1) ok = receive_mo();  // this set had no pair: take m_O first
                if (ok) ok = receive(gpair + NP - 1);
                if (!ok) break;
            }
            // -------------------------------------------------------------- epilogue
            // Row r's O is the sum of lanes r (P_hi parts) and r + 64 (P_lo parts).
            // This thread finalizes 32 columns; it hands the partner its lane's share
            // of the partner's 32 columns and of the denominator through the
            // partner's P tile (free: every P V of the unit has completed).
            ok = __all_sync(0xffffffffu, wait_bar(o_full, c & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            uint32_t oa[32], ob[32];
            tc_ld_32x32b_x32(tmem + lane_base + kGdColO + c_lo, oa);
            tc_ld_32x32b_x32(tmem + lane_base + kGdColO + c_send, ob);
            const uint32_t l_bits = tc_ld_32x32b_x1(tmem + lane_base + kGdColO + 128);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);  // the next unit's first P V may overwrite O
            {
                const uint32_t xdst = p_base + (2 * set + 1 - half) * S::kPTile;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    sts128(xdst + r * 128 + ((q ^ swz) << 4), ob[4 * q], ob[4 * q + 1], ob[4 * q + 2], ob[4 * q + 3]);
                sts32(xdst + 64 * 128 + r * 4, l_bits);
            }
            ok = meet();
            if (!ok) break;
            const float l_own = __uint_as_float(l_bits);
            {
                const uint32_t xsrc = p_base + (2 * set + half) * S::kPTile;
                const float l = l_own + __uint_as_float(lds32(xsrc + 64 * 128 + r * 4));
                const bool anyk = l > 0.f;
                const float inv = anyk ? 1.f / l : 0.f;
                float ov[32];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint4 xv = lds128(xsrc + r * 128 + ((q ^ swz) << 4));
                    ov[4 * q] = (__uint_as_float(oa[4 * q]) + __uint_as_float(xv.x)) * inv;
                    ov[4 * q + 1] = (__uint_as_float(oa[4 * q + 1]) + __uint_as_float(xv.y)) * inv;
                    ov[4 * q + 2] = (__uint_as_float(oa[4 * q + 2]) + __uint_as_float(xv.z)) * inv;
                    ov[4 * q + 3] = (__uint_as_float(oa[4 * q + 3]) + __uint_as_float(xv.w)) * inv;
                }
                // O and l are both relative to m_O = m_w - e (log2 units).
                const float lse2 = anyk ? log2f(l) - mneg - static_cast<float>(e) : -INFINITY;
                finish(u, ov, lse2);
            }
            // All four owners of these rows are done with the unit (its m_O slot).
            __syncwarp();
            if (lane == 0) mbar_arrive(&ue_bar[grp]);
            ok = __all_sync(0xffffffffu, wait_bar(&ue_bar[grp], c & 1, abort_flag, p.status));
            if (!ok) break;
            gpair += NP;
            ++c;
        }
    }
    teardown_tmem(warp == kGdMmaWarp, tmem, kGdTmemCols);
}

// Merge of the cut sequences of a persistent decode kernel's direct-output call
// with num_splits >= 2 (at most 64 query rows per KV head). One CTA per
// sequence (b, h_kv) reads the piece count the decode kernel recorded for it
// (0: written whole) and merges the pieces of a cut sequence. Thread (row r,
// quarter q) merges channels 32q .. 32q+31 of row r:
//     O = sum_s 2^(lse2_s - m) O_s / sum_s 2^(lse2_s - m),  m = max_s lse2_s.
__global__ void __launch_bounds__(256) qk4v8_cut_merge_kernel(const AttnParams p) {
    const int b = static_cast<int>(blockIdx.x) / p.Hkv, h = static_cast<int>(blockIdx.x) % p.Hkv;
    const int np = p.piece_counts[blockIdx.x];
    const int R = p.G * p.Sq, nq = p.Sq;
    const int r = threadIdx.x >> 2, c0 = (threadIdx.x & 3) * 32;
    if (np < 2 || r >= R) return;
    const int h_q = h * p.G + r / nq, tq = r % nq;
    const int64_t orow = (static_cast<int64_t>(b) * p.Hq + h_q) * nq + tq;
    const int64_t base = orow * p.num_splits;
    // Two pieces at a time, their lse and O loads issued together, with a
    // running max and sum over the pieces.
    float m = -INFINITY, wsum = 0.f;
    float acc[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) acc[k] = 0.f;
    for (int q0 = 0; q0 < np; q0 += 2) {
        const bool two = q0 + 1 < np;
        const float l0 = p.ws_lse[base + q0];
        const float l1 = two ? p.ws_lse[base + q0 + 1] : -INFINITY;
        const float4 *s0 = reinterpret_cast<const float4 *>(p.ws_o + (base + q0) * 128 + c0);
        const float4 *s1 = reinterpret_cast<const float4 *>(p.ws_o + (base + q0 + (two ? 1 : 0)) * 128 + c0);
        float4 x0[8], x1[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            x0[k] = s0[k];
            x1[k] = s1[k];
        }
        const float mn = fmaxf(m, fmaxf(l0, l1));
        if (mn == -INFINITY) continue;
        const float a = exp2f(m - mn), w0 = exp2f(l0 - mn), w1 = exp2f(l1 - mn);
        wsum = wsum * a + w0 + w1;
        m = mn;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            acc[4 * k] = acc[4 * k] * a + w0 * x0[k].x + w1 * x1[k].x;
            acc[4 * k + 1] = acc[4 * k + 1] * a + w0 * x0[k].y + w1 * x1[k].y;
            acc[4 * k + 2] = acc[4 * k + 2] * a + w0 * x0[k].z + w1 * x1[k].z;
            acc[4 * k + 3] = acc[4 * k + 3] * a + w0 * x0[k].w + w1 * x1[k].w;
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((static_cast<int64_t>(b) * nq + tq) * p.Hq + h_q) * 128 + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t w4[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const __nv_bfloat162 v2 = __floats2bfloat162_rn(acc[8 * q + 2 * kk] * inv, acc[8 * q + 2 * kk + 1] * inv);
            w4[kk] = *reinterpret_cast<const uint32_t *>(&v2);
        }
        dst[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    if (c0 == 0 && p.lse) p.lse[orow] = wsum > 0.f ? (m + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
}

cudaError_t launch_gqa_decode(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p,
                              cudaStream_t stream) {
    constexpr int kMaxDevices = 64;
    static bool configured[kMaxDevices] = {};
    static int sm_count[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int sms = dev < kMaxDevices ? sm_count[dev] : 0;
    if (dev >= kMaxDevices || !configured[dev]) {
        e = cudaFuncSetAttribute(qk4v8_gqa_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GdSmem::kBytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(qk4v8_gqa_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GdSmem::kBytes);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) {
            sm_count[dev] = sms;
            configured[dev] = true;
        }
    }
    // Persistent: one CTA per SM (shared memory and the 512 TMEM columns allow no
    // more); the kernel schedules the work over the grid itself.
    if (p.window > 0 || p.block_table || p.v_fp4)
        qk4v8_gqa_decode_kernel<true><<<sms, kGdThreads, GdSmem::kBytes, stream>>>(tk, tv, p);
    else
        qk4v8_gqa_decode_kernel<false><<<sms, kGdThreads, GdSmem::kBytes, stream>>>(tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess || !p.direct_out || p.num_splits < 2) return e;
    return launch_cut_merge(p, stream);
}

cudaError_t launch_cut_merge(const AttnParams &p, cudaStream_t stream) {
    qk4v8_cut_merge_kernel<<<p.B * p.Hkv, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace qk4v8
