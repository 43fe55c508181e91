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
// warp covers NC query rows. Rows share a reference max m that moves only when
// a score exceeds it by 2^8 (one barrier vote of the softmax threads per tile).
// So the common path needs no reduction, and p = 2^(s - m) <= 256.
// P_hi = E4M3(p), P_lo = E4M3((p - P_hi) * 32): about 8 significant bits. The
// denominator sums P_hi + P_lo exactly as the MMA sees them.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer,
// warps 2.. softmax and epilogue (4 per column group of NC rows).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pipeline.cuh"
#include "ptx.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

namespace {

constexpr float kTauD = 8.0f;
constexpr int kEMaxD = 64;
// Stages of the G*nq <= 16 instantiation, small enough for two CTAs per SM.
constexpr int kDecodeSmallStages = 3;  // largest P scale exponent before O itself is rescaled
constexpr uint32_t kPhiScaleWord = 0x7F7F7F7Fu;  // E8M0 2^0 for P_hi rows
constexpr uint32_t kPloScaleWord = 0x7A7A7A7Au;  // E8M0 2^-5 for P_lo rows
constexpr int kBarVote = 1, kBarSlow = 2, kBarEpi = 3, kBarAbort = 4;

template <int NT, int NC, int ST>
struct DecodeLayout {
    static constexpr int kStages = ST;             // K/V pipeline stages
    static constexpr int kCG = NT / NC;            // column groups
    static constexpr int kSoftmaxWarps = 4 * kCG;
    static constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
    static constexpr int kThreads = 64 + kSoftmaxThreads;
    static constexpr int kQ = 0;  // NT rows x 64 B, 64-byte swizzle (8 KB reserved)
    static constexpr int kK = 8192;
    static constexpr int kKBytes = 128 * 64;
    static constexpr int kV = kK + ST * kKBytes;
    static constexpr int kVBytes = 128 * 128;
    static constexpr int kP = kV + ST * kVBytes;  // 2 buffers of [P_hi rows; P_lo rows] x 128 B
    static constexpr int kPBytes = 2 * NT * 128;
    static constexpr int kSfQ = kP + 2 * kPBytes;
    static constexpr int kSfK = kSfQ + 512;
    static constexpr int kSfV = kSfK + ST * 512;
    static constexpr int kSfP = kSfV + ST * 512;  // one P scale atom per P buffer
    static constexpr int kRed = kSfP + 1024;      // [column group][quarter][NC] floats
    static constexpr int kLsum = kRed + 2048;     // [column group][quarter][NC] floats
    static constexpr int kAlpha = kLsum + 2048;   // [softmax warp][NC] floats
    static constexpr int kLim = kAlpha + 2048;    // [NT] int: exclusive key bound per query row
    static constexpr int kEoff = kLim + 256;      // [softmax warp][NC] int: P scale exponent per row
    static constexpr int kBar = kEoff + 2048;
    static constexpr int kNumBars = 2 * ST + 11;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16 + 1024;
    // TMEM columns: S^T x2 [0, 2NT), O^T [2NT, 4NT), then scale factors:
    // Q at 4NT, K x2 at 4NT+4, V x2 at 4NT+12, P x2 at 4NT+20.
    static constexpr uint32_t kColO = 2 * NT;
    static constexpr uint32_t kColSfQ = 4 * NT;
    static constexpr uint32_t kTmemCols = 4 * NT + 28 <= 128 ? 128 : (4 * NT + 28 <= 256 ? 256 : 512);
    static_assert(kCG * 4 * NC * 4 <= 2048, "exchange buffers");
    static_assert(kSoftmaxWarps * NC * 4 <= 2048, "rescale buffer");
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

__device__ __forceinline__ uint16_t cvt_e4m3x2_from_h2(uint32_t h2) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(r) : "r"(h2));
    return r;
}

__device__ __forceinline__ void st_u8(uint8_t *base, int off, uint32_t v) {
    base[off] = static_cast<uint8_t>(v);
}

}  // namespace

template <int NT, int NC, int ST, int MINB>
__global__ void __launch_bounds__(DecodeLayout<NT, NC, ST>::kThreads, MINB)
    qk4v8_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                        const AttnParams p) {
    using Lay = DecodeLayout<NT, NC, ST>;
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
    const int tile_begin = split * p.split_tiles;
    const int tile_end = imin(tile_begin + p.split_tiles, n_tiles);
    const int T = tile_end - tile_begin;

    auto partial_row = [&](int n) -> int64_t {
        const int h = h_kv * p.G + n / nq;
        const int t = n % nq;
        return ((static_cast<int64_t>(b) * p.Hq + h) * nq + t) * p.num_splits + split;
    };

    if (T <= 0 || (p.status && *reinterpret_cast<const volatile int32_t *>(p.status) != 0)) {
        // A split with no key: O = 0 and lse2 = -inf for every query row.
        if (warp >= 2) {
            for (int idx = threadIdx.x - 64; idx < R * 32; idx += kSoftmaxThreads) {
                const int n = idx >> 5, c4 = idx & 31;
                const int64_t row = partial_row(n);
                reinterpret_cast<float4 *>(p.ws_o + row * 128)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (c4 == 0) p.ws_lse[row] = -INFINITY;
            }
        }
        return;
    }

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::kBar);
    uint64_t *kv_full = bars;
    uint64_t *kv_empty = bars + kStagesD;
    uint64_t *q_full = bars + 2 * kStagesD;
    uint64_t *patch = q_full + 1;
    uint64_t *s_full = q_full + 2;   // [2]
    uint64_t *s_free = q_full + 4;   // [2]
    uint64_t *p_full = q_full + 6;   // [2]
    uint64_t *pv_done = q_full + 8;  // [2]
    uint64_t *o_final = q_full + 10;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::kMisc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + Lay::kMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesD; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(patch, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], Lay::kSoftmaxWarps);
            mbar_init(&p_full[s], Lay::kSoftmaxWarps);
            mbar_init(&pv_done[s], 1);
        }
        mbar_init(o_final, 1);
        *abort_flag = 0;
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
        // Q^T operand: row n < R is query head h_kv*G + n/nq at token n%nq; rows
        // R..NT-1 are zero.
        for (int c = lane; c < NT * 4; c += 32) {
            const int n = c >> 2, j = c & 3;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (n < R) {
                const int h = h_kv * p.G + n / nq, t = n % nq;
                val = *reinterpret_cast<const uint4 *>(
                    p.q_codes + ((static_cast<int64_t>(b) * p.Hq + h) * p.q_cap + t) * 64 + j * 16);
            }
            *reinterpret_cast<uint4 *>(smem + Lay::kQ + n * 64 + ((j ^ ((n >> 1) & 3)) << 4)) = val;
        }
        for (int n = lane; n < 128; n += 32) {
            uint32_t scw = 0;
            if (n < R) {
                const int h = h_kv * p.G + n / nq, t = n % nq;
                scw = *reinterpret_cast<const uint32_t *>(
                    p.q_scales + ((static_cast<int64_t>(b) * p.Hq + h) * (p.q_cap / 128) + t / 128) * 512 +
                    (t & 31) * 16 + ((t & 127) >> 5) * 4);
            }
            *reinterpret_cast<uint32_t *>(smem + Lay::kSfQ + (n & 31) * 16 + (n >> 5) * 4) = scw;
            // P scale atoms: rows [0, NT) are P_hi (2^0), rows [NT, 2NT) P_lo (2^-5);
            // the softmax raises a row's bytes when its reference max moves.
            const uint32_t pw = n < NT ? kPhiScaleWord : kPloScaleWord;
            *reinterpret_cast<uint32_t *>(smem + Lay::kSfP + (n & 31) * 16 + (n >> 5) * 4) = pw;
            *reinterpret_cast<uint32_t *>(smem + Lay::kSfP + 512 + (n & 31) * 16 + (n >> 5) * 4) = pw;
        }
        // P^T buffers start at zero; rows of absent queries are never written again.
        for (int c = lane; c < 2 * Lay::kPBytes / 16; c += 32)
            reinterpret_cast<uint4 *>(smem + Lay::kP)[c] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && !p.test_stall) mbar_arrive(q_full);

        const int kvh = b * p.Hkv + h_kv;
        const int nblk = p.kv_cap / 128;
        int issued = 0;
        for (int it = 0; it < T; ++it) {
            const int tile = tile_begin + it;
            const int st = it % kStagesD;
            const uint32_t ph = (it / kStagesD) & 1;
            bool ok = wait_bar(&kv_empty[st], ph ^ 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&kv_full[st], Lay::kKBytes + Lay::kVBytes + 1024);
                tma_load_3d(smem + Lay::kK + st * Lay::kKBytes, &tmap_k, 0, tile * 128, kvh, &kv_full[st]);
                tma_load_3d(smem + Lay::kV + st * Lay::kVBytes, &tmap_v, tile * 128, 0, kvh, &kv_full[st]);
                const int64_t atom = (static_cast<int64_t>(kvh) * nblk + tile) * 512;
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
                for (int c = lane; c < 128 * 8; c += 32) {
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
        if (lane == 0) {
            bool ok = wait_bar(q_full, 0, abort_flag, p.status);
            if (ok) {
                tc_fence_after();
                const uint32_t sb = smem_u32(smem);
                constexpr uint32_t kIdQK = idesc_d(1u, NT);      // E2M1 x E2M1, N = NT
                constexpr uint32_t kIdPV = idesc_d(0u, 2 * NT);  // E4M3 x E4M3, N = 2 NT
                // Descriptors for stage 0 / buffer 0; other stages are fixed
                // offsets of the 14-bit start-address field (in 16-byte units).
                const uint64_t dQ = smem_desc(sb + Lay::kQ, 16, 512, 4);
                const uint64_t dK0 = smem_desc(sb + Lay::kK, 16, 512, 4);
                const uint64_t dV0 = smem_desc(sb + Lay::kV, 16, 1024, 2);
                const uint64_t dP0 = smem_desc(sb + Lay::kP, 16, 1024, 2);
                const uint64_t dSfK0 = smem_desc(sb + Lay::kSfK, 0, 128, 0);
                const uint64_t dSfV0 = smem_desc(sb + Lay::kSfV, 0, 128, 0);
                tc_cp_32x128b_warpx4(tmem + Lay::kColSfQ, smem_desc(sb + Lay::kSfQ, 0, 128, 0));
                const uint64_t dSfP0 = smem_desc(sb + Lay::kSfP, 0, 128, 0);
                const uint32_t tO = tmem + Lay::kColO;
                const uint32_t tSfQ = tmem + Lay::kColSfQ;
                auto issue_pv = [&](int j) -> bool {
                    if (!wait_bar(&p_full[j & 1], (j >> 1) & 1, abort_flag, p.status)) return false;
                    tc_fence_after();
                    const int st = j % kStagesD;
                    const uint32_t tSfV = tmem + col_sf_v_d(NT, j & 1);
                    const uint32_t tSfP = tmem + col_sf_p_d(NT, j & 1);
                    tc_cp_32x128b_warpx4(tSfV, dSfV0 + static_cast<uint64_t>(st * 32));
                    tc_cp_32x128b_warpx4(tSfP, dSfP0 + static_cast<uint64_t>((j & 1) * 32));
                    const uint64_t dV = dV0 + static_cast<uint64_t>(st * (Lay::kVBytes >> 4));
                    const uint64_t dP = dP0 + static_cast<uint64_t>((j & 1) * (Lay::kPBytes >> 4));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tO, dV + 2 * k, dP + 2 * k, sf_id_d(kIdPV, k), tSfV | (k << 30), tSfP | (k << 30),
                                    (j > 0 || k > 0) ? 1u : 0u);
                    tc_commit(&pv_done[j & 1]);
                    tc_commit(&kv_empty[st]);
                    return true;
                };
                for (int it = 0; it < T && ok; ++it) {
                    const int st = it % kStagesD;
                    const int sbuf = it & 1;
                    ok = wait_bar(&kv_full[st], (it / kStagesD) & 1, abort_flag, p.status);
                    if (ok && last_partial && it == T - 1) ok = wait_bar(patch, 0, abort_flag, p.status);
                    if (ok) ok = wait_bar(&s_free[sbuf], ((it >> 1) & 1) ^ 1, abort_flag, p.status);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t tSfK = tmem + col_sf_k_d(NT, sbuf);
                    tc_cp_32x128b_warpx4(tSfK, dSfK0 + static_cast<uint64_t>(st * 32));
                    const uint64_t dK = dK0 + static_cast<uint64_t>(st * (Lay::kKBytes >> 4));
                    const uint32_t tS = tmem + static_cast<uint32_t>(NT * sbuf);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc_mma_mxf4(tS, dK + 2 * kk, dQ + 2 * kk, sf_id_d(kIdQK, 2 * kk), tSfK | ((2u * kk) << 30),
                                    tSfQ | ((2u * kk) << 30), kk > 0 ? 1u : 0u);
                    tc_commit(&s_full[sbuf]);
                    if (it >= 1) ok = issue_pv(it - 1);
                }
                if (ok) ok = issue_pv(T - 1);
                if (ok) tc_commit(o_final);
            }
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
        float *red = reinterpret_cast<float *>(smem + Lay::kRed);
        float *lsum = reinterpret_cast<float *>(smem + Lay::kLsum);
        float *alpha_s = reinterpret_cast<float *>(smem + Lay::kAlpha) + sw * NC;  // O rescale factors
        // Byte offset of (row c0 + i, token jt) in a P^T buffer, less i * 128:
        // the 128-byte swizzle puts token jt of row n in chunk (jt/16) ^ (n%8),
        // and c0 is a multiple of 8.
        const int pbase = c0 * 128 + (jt & 15);
        const int pchunk = jt >> 4;
        // Per query row: the reference max m used for p = 2^(s - m) (kept as -m,
        // +inf while the row has seen no key), and e = m - m_O, the integer
        // exponent by which m has moved above the reference m_O of the O
        // accumulator. P's E8M0 row scale carries 2^e, so O never has to be
        // rescaled while e <= kEMaxD. lacc is this thread's share of the row sum,
        // relative to m.
        float m_neg[NC];
        float lacc[NC];
        int *e_off = reinterpret_cast<int *>(smem + Lay::kEoff) + sw * NC;  // this warp's copy
#pragma unroll
        for (int i = 0; i < NC; ++i) {
            m_neg[i] = INFINITY;
            lacc[i] = 0.f;
        }
        if (lane < NC) e_off[lane] = 0;
        __syncwarp();
        int sf_dirty = 0;  // P buffers whose scale atom still holds an old e
        const float sc = p.scale_log2;
        // Key bound of each query row: L, or L - nq + t + 1 for token t of a causal
        // verify block. Tabulated once so the per-tile loop needs no division.
        int *lim_s = reinterpret_cast<int *>(smem + Lay::kLim);
        if (sw == 0)
            for (int n = lane; n < NT; n += 32) lim_s[n] = p.causal ? imin(L, L - nq + (n % nq) + 1) : L;
        bar_sync(kBarEpi, kSoftmaxThreads);
        bool ok = true;
        for (int it = 0; it < T; ++it) {
            const int sbuf = it & 1;
            ok = wait_bar(&s_full[sbuf], (it >> 1) & 1, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
            const uint32_t tS = tmem + lane_base + static_cast<uint32_t>(NT * sbuf + c0);
            uint32_t sraw[NC];
            if (ok) {
                tc_fence_after();
                tmem_load_cols<NC>(tS, sraw);
                tc_wait_ld();
            }

            const int tok = (tile_begin + it) * 128 + jt;
            // Every row may see this key unless it lies past L, or in the last
            // nq-1 positions where query t of the verify block stops at L - nq + t.
            const bool all_rows = ok && tok < L - (p.causal ? nq - 1 : 0);
            float u[NC];  // s * scale - m (log2 units); -inf when the key is masked
            float umax = -INFINITY;
            if (all_rows) {
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    u[i] = i < nv ? fmaf(__uint_as_float(sraw[i]), sc, m_neg[i]) : -INFINITY;
                    umax = fmaxf(umax, u[i]);
                }
            } else {
                const bool any_key = ok && tok < L;
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    const bool valid = any_key && i < nv && tok < lim_s[c0 + i];
                    u[i] = valid ? fmaf(__uint_as_float(sraw[i]), sc, m_neg[i]) : -INFINITY;
                    umax = fmaxf(umax, u[i]);
                }
            }
            // One vote per tile. An abort raised anywhere in the CTA also takes the
            // slow branch, where a second vote makes the exit collective, so no
            // softmax warp is left waiting at a named barrier.
            const bool need = bar_red_or(kBarVote, kSoftmaxThreads, umax > kTauD || *abort_flag != 0);
            if (!need) {
                // S buffer `sbuf` is next written by S(it+2), issued after this tile's P.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[sbuf]);
            } else {
                if (bar_red_or(kBarAbort, kSoftmaxThreads, *abort_flag != 0)) {
                    ok = false;
                    break;
                }
                // Exact per-row maximum of this tile's scaled scores (reloaded from
                // TMEM, so the raw scores need not stay live), then move m.
                uint32_t sre[NC];
                tc_fence_after();
                tmem_load_cols<NC>(tS, sre);
                tc_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[sbuf]);
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    const float x = u[i] == -INFINITY ? -INFINITY : __uint_as_float(sre[i]) * sc;
                    const float mx = warp_max_f32(x);
                    if (lane == i) red[(cg * 4 + quarter) * NC + i] = mx;
                }
                bar_sync(kBarSlow, kSoftmaxThreads);
                bool changed = false, over = false;
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    float tmax = red[(cg * 4 + 0) * NC + i];
#pragma unroll
                    for (int q = 1; q < 4; ++q) tmax = fmaxf(tmax, red[(cg * 4 + q) * NC + i]);
                    float a = 1.f;
                    if (m_neg[i] == INFINITY) {
                        // First key of the row: it fixes m_O = m.
                        if (tmax > -INFINITY) m_neg[i] = -tmax;
                    } else if (tmax + m_neg[i] > kTauD) {
                        // Move m up by a whole number of binades, so the change is
                        // an exact power of two in P's scale.
                        const int de = static_cast<int>(ceilf(tmax + m_neg[i]));
                        m_neg[i] -= static_cast<float>(de);
                        const int ne = e_off[i] + de;
                        __syncwarp();
                        if (lane == 0) e_off[i] = ne;
                        a = de < 126 ? __uint_as_float(static_cast<uint32_t>(127 - de) << 23) : 0.f;
                        changed = true;
                        over |= ne > kEMaxD;
                    }
                    lacc[i] *= a;
                    if (u[i] != -INFINITY) u[i] = fmaf(__uint_as_float(sre[i]), sc, m_neg[i]);
                }
                __syncwarp();
                if (changed) sf_dirty = 2;
                // Past kEMaxD binades O itself is brought to the current reference:
                // O *= 2^-e once PV(it-1) is done, and e restarts at 0.
                if (__any_sync(0xffffffffu, over)) {
                    __syncwarp();
                    for (int i = 0; i < NC; ++i) {
                        const int ee = e_off[i] > kEMaxD ? e_off[i] : 0;
                        __syncwarp();
                        if (lane == 0) {
                            alpha_s[i] = ee < 126 ? __uint_as_float(static_cast<uint32_t>(127 - ee) << 23) : 0.f;
                            if (ee) e_off[i] = 0;
                        }
                    }
                    __syncwarp();
                    if (it >= 1) {
                        bool okw = wait_bar(&pv_done[(it - 1) & 1], ((it - 1) >> 1) & 1, abort_flag, p.status);
                        if (__all_sync(0xffffffffu, okw)) {
                            tc_fence_after();
                            uint32_t ohi[NC], olo[NC];
                            tmem_load_cols<NC>(tmem + lane_base + Lay::kColO + c0, ohi);
                            tmem_load_cols<NC>(tmem + lane_base + Lay::kColO + NT + c0, olo);
                            tc_wait_ld();
#pragma unroll
                            for (int c = 0; c < NC; ++c) {
                                const float a = alpha_s[c];
                                ohi[c] = __float_as_uint(__uint_as_float(ohi[c]) * a);
                                olo[c] = __float_as_uint(__uint_as_float(olo[c]) * a);
                            }
                            tmem_store_cols<NC>(tmem + lane_base + Lay::kColO + c0, ohi);
                            tmem_store_cols<NC>(tmem + lane_base + Lay::kColO + NT + c0, olo);
                            tc_wait_st();
                        }
                    }
                    sf_dirty = 2;
                }
            }
            // P buffer `sbuf` was last read by PV(it-2).
            if (it >= 2) {
                bool okw = wait_bar(&pv_done[sbuf], ((it >> 1) & 1) ^ 1, abort_flag, p.status);
                (void)__all_sync(0xffffffffu, okw);
            }
            uint8_t *pb = smem + Lay::kP + sbuf * Lay::kPBytes;
            if (sf_dirty > 0) {
                // This buffer's scale atom: byte `quarter` (this warp's 32 keys) of
                // rows c0+i (P_hi, 2^e) and NT+c0+i (P_lo, 2^(e-5)).
                if (lane == 0) {
                    uint8_t *atom = smem + Lay::kSfP + sbuf * 512;
#pragma unroll
                    for (int i = 0; i < NC; ++i) {
                        const int n = c0 + i, nl = NT + c0 + i;
                        atom[(n & 31) * 16 + (n >> 5) * 4 + quarter] = static_cast<uint8_t>(127 + e_off[i]);
                        atom[(nl & 31) * 16 + (nl >> 5) * 4 + quarter] = static_cast<uint8_t>(122 + e_off[i]);
                    }
                }
                --sf_dirty;
            }
#pragma unroll
            for (int i = 0; i < NC; i += 2) {
                if (i >= nv) break;
                const float p0 = exp2_approx(u[i]);
                const float p1 = exp2_approx(u[i + 1]);
                const uint16_t h2 = cvt_e4m3x2(p0, p1);
                const uint32_t hv = cvt_e4m3x2_to_f16x2(h2);
                const __half2 ph = __floats2half2_rn(p0, p1);
                const __half2 r = __hmul2(__hsub2(ph, *reinterpret_cast<const __half2 *>(&hv)),
                                          __float2half2_rn(32.f));
                const uint16_t l2 = cvt_e4m3x2_from_h2(*reinterpret_cast<const uint32_t *>(&r));
                const uint32_t lv = cvt_e4m3x2_to_f16x2(l2);
                const __half2 pt = __hfma2(*reinterpret_cast<const __half2 *>(&lv), __float2half2_rn(0.03125f),
                                           *reinterpret_cast<const __half2 *>(&hv));
                const float2 ptf = __half22float2(pt);
                lacc[i] += ptf.x;
                lacc[i + 1] += ptf.y;
                const int o0 = pbase + ((pchunk ^ (i & 7)) << 4) + i * 128;
                const int o1 = pbase + ((pchunk ^ ((i + 1) & 7)) << 4) + (i + 1) * 128;
                st_u8(pb, o0, h2);
                st_u8(pb, o0 + NT * 128, l2);
                if (i + 1 < nv) {
                    st_u8(pb, o1, h2 >> 8);
                    st_u8(pb, o1 + NT * 128, l2 >> 8);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[sbuf]);
        }
        // ----------------------------------------------------------------- epilogue
        if (ok) {
            ok = wait_bar(o_final, 0, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
        }
        // Row denominators: sum the per-token partial sums over the 128 lanes.
#pragma unroll
        for (int i = 0; i < NC; ++i) {
            float v = lacc[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) lsum[(cg * 4 + quarter) * NC + i] = v;
        }
        bar_sync(kBarEpi, kSoftmaxThreads);
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
                    const float l = lsum[(cg * 4 + 0) * NC + i] + lsum[(cg * 4 + 1) * NC + i] +
                                    lsum[(cg * 4 + 2) * NC + i] + lsum[(cg * 4 + 3) * NC + i];
                    const bool any = l > 0.f && m_neg[i] < INFINITY;
                    const int64_t row = partial_row(c0 + i);
                    // O is relative to m_O = m - e: divide by l * 2^e.
                    const float inv = any ? __uint_as_float(static_cast<uint32_t>(127 - e_off[i]) << 23) / l : 0.f;
                    p.ws_o[row * 128 + jt] = (__uint_as_float(ohi[e]) + __uint_as_float(olo[e])) * inv;
                    if (jt == 0) p.ws_lse[row] = any ? log2f(l) - m_neg[i] : -INFINITY;
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

template <int NT, int NC, int ST, int MINB>
static cudaError_t launch_nt(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, int grid,
                             cudaStream_t stream) {
    using Lay = DecodeLayout<NT, NC, ST>;
    constexpr int kMaxDevices = 64;
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !configured[dev]) {
        e = cudaFuncSetAttribute(qk4v8_decode_kernel<NT, NC, ST, MINB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Lay::kBytes);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) configured[dev] = true;
    }
    qk4v8_decode_kernel<NT, NC, ST, MINB><<<grid, Lay::kThreads, Lay::kBytes, stream>>>(tk, tv, p);
    return cudaGetLastError();
}

cudaError_t launch_decode(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, int grid,
                          cudaStream_t stream) {
    const int R = p.G * p.Sq;
    if (R <= 16) return launch_nt<16, 16, kDecodeSmallStages, 2>(tk, tv, p, grid, stream);
    if (R <= 32) return launch_nt<32, 16, 6, 1>(tk, tv, p, grid, stream);
    return launch_nt<64, 16, 6, 1>(tk, tv, p, grid, stream);
}

}  // namespace qk4v8
