// QK4V8 attention on sm_100a: block-scaled tcgen05 MMAs with TMEM accumulators.
//
// MpFA QK4V8 article (mhpn.cn), sections 2.3, 3.3, 5.1: attention runs block
// by block with an online softmax. Each block's 4-bit QK^T scores are
// dequantized as soon as they are computed and feed an FP32 softmax. P is then
// multiplied with the 8-bit V into an FP32 accumulator, and the dequantization
// multiply is folded into the tensor-core MMA. Here the folding is exact:
//  - S = Q K^T runs as tcgen05.mma kind::mxf4 (E2M1 x E2M1) with the E8M0
//    group-of-32 scales of Q and K applied by the hardware.
//  - O += P V runs as tcgen05.mma kind::mxf8f6f4 (E4M3 x E4M3). Its scales
//    are the V scales (per channel, per 32 tokens) and a per-row,
//    per-32-token E8M0 scale chosen for P.
//  - P is split into two E4M3 terms, P = P_hi + P_lo, each with its own
//    scales, so the 8-bit P carries about 8 significant bits.
//  - V is extended with a row of ones, so column 128 of the O accumulator is
//    the softmax denominator sum_j P_hi + P_lo, accumulated by the same MMA.
//
// One CTA computes one work unit: 128 query rows against one KV head. The
// library launches it for split-KV decode with 65..128 query rows per KV head
// (the swap-AB decode kernel covers up to 64, the prefill kernel prefill):
//  - Decode unit: the G*nq query rows of a GQA group against one contiguous
//    split of the KV cache. Rows go round-robin over the four TMEM lane quarters.
//  - The kDecode = false form (one query head, 128 consecutive query tokens) is
//    kept in the template but not instantiated.
// Warp roles (192 threads):
//  - warp 0: TMA producer (Q gather, K/V tiles, scale atoms; ragged-tile cleanup)
//  - warp 1: TMEM allocator and single-thread MMA issuer
//  - warps 2-5: softmax, one TMEM lane (one query row) per thread; epilogue
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pipeline.cuh"
#include "ptx.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

namespace {

constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr float kTau = 8.0f;  // lazy rescaling: the running max moves only when a score exceeds it by 2^8

// Shared memory map (byte offsets from a 1024-aligned base).
constexpr int kQOff = 0;                                // Q tile: 128 rows x 64 B, 64-byte swizzle
constexpr int kKOff = kQOff + 128 * 64;                 // K tiles: 128 tokens x 64 B, 64-byte swizzle
constexpr int kKBytes = 128 * 64;
constexpr int kVOff = kKOff + kStages * kKBytes;        // V tiles: 144 rows x 128 B, 128-byte swizzle
constexpr int kVRows = 144;                             // 128 channels, a ones row, 15 zero rows
constexpr int kVBytes = kVRows * 128;
constexpr int kVTmaBytes = 128 * 128;
constexpr int kPhiOff = kVOff + kStages * kVBytes;      // P_hi: 128 rows x 128 B, 128-byte swizzle
constexpr int kPloOff = kPhiOff + 128 * 128;            // P_lo
constexpr int kSfQOff = kPloOff + 128 * 128;            // 512-byte scale atoms
constexpr int kSfKOff = kSfQOff + 512;
constexpr int kSfVOff = kSfKOff + kStages * 512;
constexpr int kSfPhiOff = kSfVOff + kStages * 512;
constexpr int kSfPloOff = kSfPhiOff + 512;
constexpr int kSfOneOff = kSfPloOff + 512;
constexpr int kBarOff = kSfOneOff + 512;
constexpr int kNumBars = 2 * kStages + 9;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kSmemUsed = kMiscOff + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;  // slack for aligning the base

// TMEM columns (512 allocated; one CTA per SM).
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int buf) { return 128u * buf; }  // S double buffer: 0, 128
constexpr uint32_t kColO = 256;    // 144 columns: O[:, 0:128], row sum in column 128
constexpr uint32_t kColSfQ = 400;
__device__ __forceinline__ uint32_t col_sf_k(int buf) { return 404u + 4u * buf; }
constexpr uint32_t kColSfPhi = 412;
constexpr uint32_t kColSfPlo = 416;
// V scale columns per buffer (420, 428), each followed by 4 constant columns
// holding the scale of the ones row.
__device__ __forceinline__ uint32_t col_sf_v(int buf) { return 420u + 8u * buf; }

// Instruction descriptors (kind::mxf4 / kind::mxf8f6f4 with E8M0 block scales,
// K-major A and B, FP32 accumulate), scale-factor ids added per MMA.
constexpr uint32_t idesc_base(uint32_t fmt, uint32_t n) {
    return (fmt << 7) | (fmt << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}
constexpr uint32_t kIdescQK = idesc_base(1u, 128);  // E2M1 x E2M1, N = 128 keys
constexpr uint32_t kIdescPV = idesc_base(0u, kVRows);  // E4M3 x E4M3, N = 144
__device__ __forceinline__ uint32_t with_sf_id(uint32_t idesc, uint32_t id) {
    return idesc | (id << 29) | (id << 4);
}

constexpr uint32_t kSw128 = 2, kSw64 = 4, kSwNone = 0;

struct Bars {
    uint64_t *kv_full, *kv_empty, *q_full, *patch, *s_full, *s_free, *p_full, *pv_done, *o_final;
};

struct Unit {
    int b, h_kv, h_q, q0, R, L, tile_begin, tile_end, split;
};

template <bool kDecode>
__device__ __forceinline__ Unit decode_unit(const AttnParams &p) {
    Unit u;
    if (!kDecode) {
        const int per = p.B * p.Hq;
        const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / per;  // longest (causal) first
        const int rem = static_cast<int>(blockIdx.x) % per;
        u.b = rem / p.Hq;
        u.h_q = rem % p.Hq;
        u.h_kv = u.h_q / p.G;
        u.q0 = qt * 128;
        u.R = imin(128, p.Sq - u.q0);
        u.split = 0;
        int L = p.seqlens ? p.seqlens[u.b] : p.Lk;
        u.L = imax(0, imin(L, p.kv_cap));
        int kv_end = u.L;
        if (p.causal) kv_end = imin(u.L, u.q0 + u.R + u.L - p.Sq);
        u.tile_begin = 0;
        u.tile_end = kv_end > 0 ? (kv_end + 127) / 128 : 0;
    } else {
        u.split = static_cast<int>(blockIdx.x) % p.num_splits;
        const int rem = static_cast<int>(blockIdx.x) / p.num_splits;
        u.h_kv = rem % p.Hkv;
        u.b = rem / p.Hkv;
        u.h_q = u.h_kv * p.G;
        u.q0 = 0;
        u.R = p.G * p.Sq;
        int L = p.seqlens ? p.seqlens[u.b] : p.Lk;
        u.L = imax(0, imin(L, p.kv_cap));
        const int n_tiles = (u.L + 127) / 128;
        u.tile_begin = u.split * p.split_tiles;
        u.tile_end = imin(u.tile_begin + p.split_tiles, n_tiles);
    }
    return u;
}

// Row carried by TMEM lane `lane` (0..127): query head, query token and the
// exclusive bound on its keys. Prefill rows follow the lanes directly; decode
// rows go round-robin over the four lane quarters.
struct RowInfo {
    bool valid;
    int h, i, limit;
};

template <bool kDecode>
__device__ __forceinline__ RowInfo row_info(const AttnParams &p, const Unit &u, int lane) {
    RowInfo r;
    int idx;
    if (!kDecode) {
        idx = lane;
        r.h = u.h_q;
        r.i = u.q0 + lane;
    } else {
        idx = (lane & 31) * 4 + (lane >> 5);
        r.h = u.h_kv * p.G + (p.Sq > 0 ? idx / p.Sq : 0);
        r.i = p.Sq > 0 ? idx % p.Sq : 0;
    }
    r.valid = idx < u.R;
    int lim = u.L;
    if (p.causal) lim = imin(lim, r.i + u.L - p.Sq + 1);
    r.limit = r.valid ? imax(lim, 0) : 0;
    return r;
}


// Writes the result of a row that saw no key at all.
template <bool kDecode>
__device__ __forceinline__ void write_empty_row(const AttnParams &p, const Unit &u, const RowInfo &r) {
    if (!r.valid) return;
    if (!kDecode) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((static_cast<int64_t>(u.b) * p.Sq + r.i) * p.Hq + r.h) * 128);
#pragma unroll
        for (int q = 0; q < 16; ++q) dst[q] = make_uint4(0, 0, 0, 0);
        if (p.lse) p.lse[(static_cast<int64_t>(u.b) * p.Hq + r.h) * p.Sq + r.i] = -INFINITY;
    } else {
        const int64_t row = ((static_cast<int64_t>(u.b) * p.Hq + r.h) * p.Sq + r.i) * p.num_splits + u.split;
        float4 *dst = reinterpret_cast<float4 *>(p.ws_o + row * 128);
#pragma unroll
        for (int q = 0; q < 32; ++q) dst[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        p.ws_lse[row] = -INFINITY;
    }
}

}  // namespace

template <bool kDecode>
__global__ void __launch_bounds__(kThreads, 1)
    qk4v8_attention_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                           const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const Unit u = decode_unit<kDecode>(p);
    const int T = u.tile_end - u.tile_begin;
    if (T <= 0) {
        if (warp >= 2) write_empty_row<kDecode>(p, u, row_info<kDecode>(p, u, ((warp & 3) << 5) | lane));
        return;
    }

    uint64_t *bar_base = reinterpret_cast<uint64_t *>(smem + kBarOff);
    Bars bars;
    bars.kv_full = bar_base;
    bars.kv_empty = bar_base + kStages;
    bars.q_full = bar_base + 2 * kStages;
    bars.patch = bars.q_full + 1;
    bars.s_full = bars.q_full + 2;   // [2]
    bars.s_free = bars.q_full + 4;   // [2]
    bars.p_full = bars.q_full + 6;
    bars.pv_done = bars.q_full + 7;
    bars.o_final = bars.q_full + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kMiscOff);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + kMiscOff + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.kv_empty[s], 1);
        }
        mbar_init(bars.q_full, 1);
        mbar_init(bars.patch, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars.s_full[s], 1);
            mbar_init(&bars.s_free[s], 4);
        }
        mbar_init(bars.p_full, 4);
        mbar_init(bars.pv_done, 1);
        mbar_init(bars.o_final, 1);
        // A status already set by another launch or CTA: unwind at once (every
        // wait returns false), decided once for the whole CTA.
        *abort_flag = (p.status && *reinterpret_cast<const volatile int32_t *>(p.status) != 0) ? 1u : 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // The last tile is ragged when L is not a multiple of 128 and it is in range.
    const bool last_partial = (u.L & 127) != 0 && u.tile_end == (u.L + 127) / 128;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        // Q rows into the 64-byte-swizzled A tile and the Q scale atom; rows that
        // carry no query are zero.
        uint8_t *qs = smem + kQOff;
        for (int c = lane; c < 512; c += 32) {
            const int row = c >> 2, j = c & 3;
            const RowInfo r = row_info<kDecode>(p, u, row);
            uint4 val = make_uint4(0, 0, 0, 0);
            if (r.valid)
                val = *reinterpret_cast<const uint4 *>(
                    p.q_codes + ((static_cast<int64_t>(u.b) * p.Hq + r.h) * p.q_cap + r.i) * 64 + j * 16);
            *reinterpret_cast<uint4 *>(qs + row * 64 + ((j ^ ((row >> 1) & 3)) << 4)) = val;
        }
        for (int row = lane; row < 128; row += 32) {
            const RowInfo r = row_info<kDecode>(p, u, row);
            uint32_t sc = 0;
            if (r.valid)
                sc = *reinterpret_cast<const uint32_t *>(
                    p.q_scales + ((static_cast<int64_t>(u.b) * p.Hq + r.h) * (p.q_cap / 128) + r.i / 128) * 512 +
                    (r.i & 31) * 16 + ((r.i & 127) >> 5) * 4);
            *reinterpret_cast<uint32_t *>(smem + kSfQOff + (row & 31) * 16 + (row >> 5) * 4) = sc;
        }
        // Constant operand rows: V row 128 = 1.0 (E4M3 0x38), rows 129..143 = 0,
        // and a scale atom of 2^0 bytes for those rows.
        for (int s = 0; s < kStages; ++s)
            for (int c = lane; c < 16 * 8; c += 32) {
                const int row = 128 + (c >> 3);
                const uint32_t fillv = row == 128 ? 0x38383838u : 0u;
                *reinterpret_cast<uint4 *>(smem + kVOff + s * kVBytes + row * 128 + (c & 7) * 16) =
                    make_uint4(fillv, fillv, fillv, fillv);
            }
        for (int c = lane; c < 32; c += 32)
            *reinterpret_cast<uint4 *>(smem + kSfOneOff + c * 16) =
                make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && !p.test_stall) mbar_arrive(bars.q_full);

        const int kvh = u.b * p.Hkv + u.h_kv;
        const int nblk = p.kv_cap / 128;
        int issued = 0;
        for (int it = 0; it < T; ++it) {
            const int tile = u.tile_begin + it;
            const int st = it % kStages;
            const uint32_t ph = (it / kStages) & 1;
            bool ok = wait_bar(&bars.kv_empty[st], ph ^ 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars.kv_full[st], kKBytes + kVTmaBytes + 1024);
                tma_load_3d(smem + kKOff + st * kKBytes, &tmap_k, 0, tile * 128, kvh, &bars.kv_full[st]);
                tma_load_3d(smem + kVOff + st * kVBytes, &tmap_v, 0, 0, kvh * nblk + tile, &bars.kv_full[st]);
                const int64_t atom = (static_cast<int64_t>(kvh) * nblk + tile) * 512;
                bulk_load(smem + kSfKOff + st * 512, p.k_scales + atom, 512, &bars.kv_full[st]);
                bulk_load(smem + kSfVOff + st * 512, p.v_scales + atom, 512, &bars.kv_full[st]);
            }
            issued = it + 1;
            if (last_partial && tile == u.tile_end - 1) {
                // Keys at or past L may hold anything (a reused cache). Their P is
                // zero, but a NaN code or scale would still poison O, so zero them.
                ok = wait_bar(&bars.kv_full[st], ph, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) break;
                const int jv = u.L - tile * 128;  // valid tokens in this tile, 1..127
                uint8_t *vt = smem + kVOff + st * kVBytes;
                for (int c = lane; c < 128 * 8; c += 32) {
                    const int row = c >> 3, q = c & 7;
                    if (16 * q + 16 <= jv) continue;
                    uint8_t *chunk = vt + row * 128 + ((q ^ (row & 7)) << 4);
                    for (int e = 0; e < 16; ++e)
                        if (16 * q + e >= jv) chunk[e] = 0;
                }
                uint8_t *sfv = smem + kSfVOff + st * 512;
                for (int row = lane; row < 128; row += 32)
                    for (int g = (jv + 31) / 32; g < 4; ++g) sfv[(row & 31) * 16 + (row >> 5) * 4 + g] = 0;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.patch);
            }
        }
        // Let every issued copy land before the CTA can retire.
        if (lane == 0) {
            for (int it = imax(0, issued - kStages); it < issued; ++it) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bars.kv_full[it % kStages], (it / kStages) & 1))
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            bool ok = wait_bar(bars.q_full, 0, abort_flag, p.status);
            if (ok) {
                tc_fence_after();
                const uint32_t sb = smem_u32(smem);
                auto atom_desc = [&](int off) { return smem_desc(sb + off, 0, 128, kSwNone); };
                tc_cp_32x128b_warpx4(tmem + kColSfQ, atom_desc(kSfQOff));
                tc_cp_32x128b_warpx4(tmem + col_sf_v(0) + 4, atom_desc(kSfOneOff));
                tc_cp_32x128b_warpx4(tmem + col_sf_v(1) + 4, atom_desc(kSfOneOff));
                auto issue_pv = [&](int j) -> bool {
                    if (!wait_bar(bars.p_full, j & 1, abort_flag, p.status)) return false;
                    tc_fence_after();
                    const int st = j % kStages, vb = j & 1;
                    tc_cp_32x128b_warpx4(tmem + col_sf_v(vb), atom_desc(kSfVOff + st * 512));
                    tc_cp_32x128b_warpx4(tmem + kColSfPhi, atom_desc(kSfPhiOff));
                    tc_cp_32x128b_warpx4(tmem + kColSfPlo, atom_desc(kSfPloOff));
                    const uint32_t vaddr = sb + kVOff + st * kVBytes;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tmem + kColO, smem_desc(sb + kPhiOff + 32 * k, 16, 1024, kSw128),
                                    smem_desc(vaddr + 32 * k, 16, 1024, kSw128), with_sf_id(kIdescPV, k),
                                    (tmem + kColSfPhi) | (k << 30), (tmem + col_sf_v(vb)) | (k << 30),
                                    (j > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_mxf8(tmem + kColO, smem_desc(sb + kPloOff + 32 * k, 16, 1024, kSw128),
                                    smem_desc(vaddr + 32 * k, 16, 1024, kSw128), with_sf_id(kIdescPV, k),
                                    (tmem + kColSfPlo) | (k << 30), (tmem + col_sf_v(vb)) | (k << 30), 1u);
                    tc_commit(bars.pv_done);
                    tc_commit(&bars.kv_empty[st]);
                    return true;
                };
                for (int it = 0; it < T && ok; ++it) {
                    const int st = it % kStages;
                    const int sbuf = it & 1;
                    ok = wait_bar(&bars.kv_full[st], (it / kStages) & 1, abort_flag, p.status);
                    if (ok && last_partial && it == T - 1) ok = wait_bar(bars.patch, 0, abort_flag, p.status);
                    if (ok) ok = wait_bar(&bars.s_free[sbuf], ((it >> 1) & 1) ^ 1, abort_flag, p.status);
                    if (!ok) break;
                    tc_fence_after();
                    tc_cp_32x128b_warpx4(tmem + col_sf_k(sbuf), atom_desc(kSfKOff + st * 512));
                    const uint32_t kaddr = sb + kKOff + st * kKBytes;
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc_mma_mxf4(tmem + col_s(sbuf), smem_desc(sb + kQOff + 32 * kk, 16, 512, kSw64),
                                    smem_desc(kaddr + 32 * kk, 16, 512, kSw64), with_sf_id(kIdescQK, 2 * kk),
                                    (tmem + kColSfQ) | ((2u * kk) << 30), (tmem + col_sf_k(sbuf)) | ((2u * kk) << 30),
                                    kk > 0 ? 1u : 0u);
                    tc_commit(&bars.s_full[sbuf]);
                    if (it >= 1) ok = issue_pv(it - 1);
                }
                if (ok) ok = issue_pv(T - 1);
                if (ok) tc_commit(bars.o_final);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------- softmax
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const RowInfo r = row_info<kDecode>(p, u, row);
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        uint8_t *phi = smem + kPhiOff + row * 128;
        uint8_t *plo = smem + kPloOff + row * 128;
        const int swz = row & 7;
        const int sf_off = (row & 31) * 16 + (row >> 5) * 4;
        float m_ref = -INFINITY;  // running reference max, log2 units
        bool ok = true;
        for (int it = 0; it < T; ++it) {
            const int sbuf = it & 1;
            ok = wait_bar(&bars.s_full[sbuf], (it >> 1) & 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t s[4][32];
#pragma unroll
            for (int k = 0; k < 4; ++k) tc_ld_32x32b_x32(tmem + lane_base + col_s(sbuf) + 32 * k, s[k]);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.s_free[sbuf]);
            if (p.test_dump_s && blockIdx.x == 0 && it == 0) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) p.test_dump_s[row * 128 + 32 * k + jj] = __uint_as_float(s[k][jj]);
            }

            const int tok0 = (u.tile_begin + it) * 128;
            const int jv = imax(0, imin(r.limit - tok0, 128));  // keys j < jv are allowed
            float bmax[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float mx = -INFINITY;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const float x = (32 * k + jj < jv) ? __uint_as_float(s[k][jj]) : -INFINITY;
                    mx = fmaxf(mx, x);
                }
                bmax[k] = mx * p.scale_log2;
            }
            const float tmax = fmaxf(fmaxf(bmax[0], bmax[1]), fmaxf(bmax[2], bmax[3]));
            float alpha = 1.f;
            bool rescale = false;
            if (tmax > -INFINITY) {
                if (m_ref == -INFINITY) {
                    m_ref = tmax;
                } else if (tmax > m_ref + kTau) {
                    alpha = exp2_approx(m_ref - tmax);
                    m_ref = tmax;
                    rescale = true;
                }
            }
            // P = 2^(s*scale - m_ref) as two E4M3 terms per 32-key block.
            uint32_t hiw[32], low[32];
            uint32_t sf_hi = 0, sf_lo = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float pmax = (bmax[k] > -INFINITY) ? exp2_approx(bmax[k] - m_ref) : 0.f;
                int e = static_cast<int>((__float_as_uint(pmax) >> 23) & 0xFF) - 127;
                e = e < -110 ? -110 : e;
                const int x_hi = e - 7;  // P_hi / 2^x_hi < 256
                const float f_hi = __uint_as_float(static_cast<uint32_t>(127 - x_hi) << 23);
                sf_hi |= static_cast<uint32_t>(x_hi + 127) << (8 * k);
                sf_lo |= static_cast<uint32_t>(x_hi - 5 + 127) << (8 * k);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t wh = 0, wl = 0;
#pragma unroll
                    for (int e2 = 0; e2 < 4; e2 += 2) {
                        const int j = 32 * k + 4 * q + e2;
                        const float p0 = (j < jv) ? exp2_approx(fmaf(__uint_as_float(s[k][4 * q + e2]), p.scale_log2, -m_ref)) : 0.f;
                        const float p1 = (j + 1 < jv) ? exp2_approx(fmaf(__uint_as_float(s[k][4 * q + e2 + 1]), p.scale_log2, -m_ref)) : 0.f;
                        const float y0 = p0 * f_hi, y1 = p1 * f_hi;
                        const uint16_t h2 = cvt_e4m3x2(y0, y1);
                        const uint32_t hf = cvt_e4m3x2_to_f16x2(h2);
                        const float2 hv = __half22float2(*reinterpret_cast<const __half2 *>(&hf));
                        const uint16_t l2 = cvt_e4m3x2((y0 - hv.x) * 32.f, (y1 - hv.y) * 32.f);
                        wh |= static_cast<uint32_t>(h2) << (8 * e2);
                        wl |= static_cast<uint32_t>(l2) << (8 * e2);
                    }
                    hiw[8 * k + q] = wh;
                    low[8 * k + q] = wl;
                }
            }
            // PV(it-1) must be done before P is overwritten or O is rescaled.
            if (it >= 1) {
                ok = wait_bar(bars.pv_done, (it - 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
            }
            if (__any_sync(0xffffffffu, rescale)) {
                uint32_t o[32];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    tc_ld_32x32b_x32(tmem + lane_base + kColO + 32 * k, o);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tc_st_32x32b_x32(tmem + lane_base + kColO + 32 * k, o);
                }
                uint32_t o16[16];
                tc_ld_32x32b_x16(tmem + lane_base + kColO + 128, o16);
                tc_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c) o16[c] = __float_as_uint(__uint_as_float(o16[c]) * alpha);
                tc_st_32x32b_x16(tmem + lane_base + kColO + 128, o16);
                tc_wait_st();
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                *reinterpret_cast<uint4 *>(phi + ((q ^ swz) << 4)) =
                    make_uint4(hiw[4 * q], hiw[4 * q + 1], hiw[4 * q + 2], hiw[4 * q + 3]);
                *reinterpret_cast<uint4 *>(plo + ((q ^ swz) << 4)) =
                    make_uint4(low[4 * q], low[4 * q + 1], low[4 * q + 2], low[4 * q + 3]);
            }
            *reinterpret_cast<uint32_t *>(smem + kSfPhiOff + sf_off) = sf_hi;
            *reinterpret_cast<uint32_t *>(smem + kSfPloOff + sf_off) = sf_lo;
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_full);
        }
        if (ok) {
            ok = wait_bar(bars.o_final, 0, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            tc_fence_after();
            uint32_t o[4][32];
#pragma unroll
            for (int k = 0; k < 4; ++k) tc_ld_32x32b_x32(tmem + lane_base + kColO + 32 * k, o[k]);
            uint32_t o16[16];
            tc_ld_32x32b_x16(tmem + lane_base + kColO + 128, o16);
            tc_wait_ld();
            const float l = __uint_as_float(o16[0]);
            if (r.valid) {
                const bool any = l > 0.f && m_ref > -INFINITY;
                const float inv = any ? 1.f / l : 0.f;
                const float lse2 = any ? m_ref + log2f(l) : -INFINITY;
                if (!kDecode) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        p.out + ((static_cast<int64_t>(u.b) * p.Sq + r.i) * p.Hq + r.h) * 128);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int c = 8 * q + 2 * e2;
                            const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(o[c >> 5][c & 31]) * inv,
                                                                            __uint_as_float(o[(c + 1) >> 5][(c + 1) & 31]) * inv);
                            w[e2] = *reinterpret_cast<const uint32_t *>(&v2);
                        }
                        dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    if (p.lse) p.lse[(static_cast<int64_t>(u.b) * p.Hq + r.h) * p.Sq + r.i] = lse2 * 0.6931471805599453f;
                } else {
                    const int64_t prow =
                        ((static_cast<int64_t>(u.b) * p.Hq + r.h) * p.Sq + r.i) * p.num_splits + u.split;
                    float4 *dst = reinterpret_cast<float4 *>(p.ws_o + prow * 128);
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        const int c = 4 * q;
                        dst[q] = make_float4(__uint_as_float(o[c >> 5][c & 31]) * inv,
                                             __uint_as_float(o[c >> 5][(c & 31) + 1]) * inv,
                                             __uint_as_float(o[c >> 5][(c & 31) + 2]) * inv,
                                             __uint_as_float(o[c >> 5][(c & 31) + 3]) * inv);
                    }
                    p.ws_lse[prow] = lse2;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Combine the split partials (m, l, O) of decode rows: one warp per query row.
__global__ void __launch_bounds__(256) qk4v8_decode_merge_kernel(const float *__restrict__ ws_o,
                                                                 const float *__restrict__ ws_lse, int B, int Hq,
                                                                 int nq, int splits, __nv_bfloat16 *__restrict__ out,
                                                                 float *__restrict__ lse) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int rows = B * Hq * nq;
    if (warp >= rows) return;
    const int t = warp % nq;
    const int h = (warp / nq) % Hq;
    const int b = warp / (nq * Hq);
    const float *lrow = ws_lse + static_cast<int64_t>(warp) * splits;
    float mx = -INFINITY;
    for (int s = lane; s < splits; s += 32) mx = fmaxf(mx, lrow[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (mx > -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float ls = lrow[s];
            if (ls == -INFINITY) continue;
            const float w = exp2f(ls - mx);
            wsum += w;
            const float4 v = reinterpret_cast<const float4 *>(ws_o + (static_cast<int64_t>(warp) * splits + s) * 128)[lane];
            acc.x += w * v.x;
            acc.y += w * v.y;
            acc.z += w * v.z;
            acc.w += w * v.w;
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    __nv_bfloat162 a = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 c = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 packed = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&c));
    reinterpret_cast<uint2 *>(out + ((static_cast<int64_t>(b) * nq + t) * Hq + h) * 128)[lane] = packed;
    if (lse && lane == 0)
        lse[(static_cast<int64_t>(b) * Hq + h) * nq + t] =
            wsum > 0.f ? (mx + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
}

// The 128-row kernel serves split-KV decode with more than 64 query rows per
// KV head (prefill has its own kernel).
cudaError_t launch_attention(const CUtensorMap &tmap_k, const CUtensorMap &tmap_v, const AttnParams &p, int grid,
                             cudaStream_t stream) {
    if (!p.decode) return cudaErrorInvalidValue;
    // The dynamic shared-memory limit is a per-device function attribute.
    constexpr int kMaxDevices = 64;
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !configured[dev]) {
        e = cudaFuncSetAttribute(qk4v8_attention_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) configured[dev] = true;
    }
    qk4v8_attention_kernel<true><<<grid, kThreads, kSmemBytes, stream>>>(tmap_k, tmap_v, p);
    return cudaGetLastError();
}

cudaError_t launch_decode_merge(const float *ws_o, const float *ws_lse, int B, int Hq, int nq, int splits,
                                __nv_bfloat16 *out, float *lse, cudaStream_t stream) {
    const int rows = B * Hq * nq;
    const int grid = (rows * 32 + 255) / 256;
    qk4v8_decode_merge_kernel<<<grid, 256, 0, stream>>>(ws_o, ws_lse, B, Hq, nq, splits, out, lse);
    return cudaGetLastError();
}

}  // namespace qk4v8
