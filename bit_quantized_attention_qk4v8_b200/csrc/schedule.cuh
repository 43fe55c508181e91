// Work schedule of the persistent decode kernels: which (sequence, KV head)
// key-tile ranges each CTA runs, either as fixed splits or balanced evenly over
// the grid ("stream-K"), and the iterator every role warp of a CTA walks.
#pragma once

#include <cstdint>

#include "pipeline.cuh"
#include "qk4v8_internal.h"

namespace qk4v8 {

// One piece of work: key tiles [tile_begin, tile_begin + T) of the sequence
// (b, h_kv), absolute tile indices. `whole` when the piece is the whole
// sequence; otherwise it is piece `slot` of `n_pieces`, written as a partial
// (O / l, log2-sum-exp).
struct GdUnit {
    int b, h_kv, L, tile_begin, T, slot, n_pieces;
    bool whole;
};

// Key tiles of sequence b the schedule covers: from the tile holding its first
// visible key to its last key.
__device__ __forceinline__ int gd_tiles(const AttnParams &p, int b) {
    const int L = imax(0, imin(p.seqlens[b], p.kv_cap));
    return (L + 127) / 128 - kv_window_lo(p, L) / 128;
}

// Schedule of one CTA, computed once at the start.
//   Fixed splits: units (sequence, split) blockIdx.x, +grid, ... with
//   split_tiles key tiles each.
//   Balanced ("stream-K"): the key tiles of all sequences in (b, h_kv) order
//   form one list of W tiles; CTA i takes tiles [i W / G, (i+1) W / G), so every
//   CTA gets the same work up to one tile. A sequence cut by a range boundary
//   becomes pieces in consecutive CTAs. Used for the direct-output call when
//   every range is at least one tile and no sequence can be cut into more
//   pieces than there are partial slots (num_splits). A CTA runs the first and
//   the last sequence of its range (the ones that may be cut) before the ones
//   in between, so that cut sequences are complete, and merged, early.
struct GdSched {
    int streamk;
    int b0, h0, bL, hL;   // first and last sequence of this CTA's range
    long long W, x0, x1;  // tile list length and this CTA's range [x0, x1)
    long long P0, PL;     // first tiles of those sequences in the list
};

// CTA holding tile x of the balanced list: the largest i with floor(i W / G) <= x.
__device__ __forceinline__ int gd_cta_of(long long x, long long W, int G) {
    return static_cast<int>(((x + 1) * G - 1) / W);
}

// Finds the first sequence (in (b, h) order) that is non-empty and ends past
// tile x, or (allow_empty) is empty and starts at or past x. One full warp.
// Returns false if there is none.
static __device__ __noinline__ bool gd_find(const AttnParams &p, long long x, bool allow_empty, int &b_out, int &h_out,
                                     long long &P_out) {
    const int lane = threadIdx.x & 31;
    long long P = 0;  // first tile of batch entry `base`
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        const int t = b < p.B ? gd_tiles(p, b) : 0;
        long long incl = static_cast<long long>(t) * p.Hkv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const long long Pb = P + incl - static_cast<long long>(t) * p.Hkv;
        const bool hit =
            b < p.B && ((t > 0 && Pb + static_cast<long long>(t) * p.Hkv > x) || (allow_empty && t == 0 && Pb >= x));
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            const int tb = __shfl_sync(0xffffffffu, t, src);
            const long long pb = __shfl_sync(0xffffffffu, Pb, src);
            b_out = base + src;
            h_out = (tb > 0 && x > pb) ? static_cast<int>((x - pb) / tb) : 0;
            P_out = pb + static_cast<long long>(h_out) * tb;
            return true;
        }
        P += __shfl_sync(0xffffffffu, incl, 31);
    }
    return false;
}

// Whether the balanced schedule applies: at least one tile per CTA, and no
// sequence cut into more pieces than the num_splits partial slots (a sequence
// of t tiles meets at most ceil(t / range) + 1 of the ranges).
__device__ __forceinline__ bool gd_balanced(const AttnParams &p, long long W, int tmax, int G) {
    const long long range = W / G;
    return p.num_splits >= 2 && range >= 1 && (tmax + range - 1) / range + 1 <= p.num_splits;
}

// Computed by one full warp: per-batch tile counts scanned 32 at a time.
static __device__ __noinline__ void gd_schedule(const AttnParams &p, GdSched &sc) {
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x, i = blockIdx.x;
    sc.streamk = 0;
    sc.b0 = sc.h0 = sc.bL = sc.hL = 0;
    sc.P0 = sc.PL = 0;
    sc.x0 = sc.x1 = sc.W = 0;
    if (!p.direct_out || p.num_splits < 2) return;  // fixed splits: no scan needed
    long long W = 0;
    int tmax = 0;
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        const int t = b < p.B ? gd_tiles(p, b) : 0;
        tmax = max(tmax, __reduce_max_sync(0xffffffffu, t));
        W += static_cast<long long>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(t))) * p.Hkv;
    }
    sc.W = W;
    if (!gd_balanced(p, W, tmax, G)) return;
    sc.streamk = 1;
    sc.x0 = static_cast<long long>(i) * W / G;
    const long long x1 = static_cast<long long>(i + 1) * W / G;
    // The last CTA also takes the empty sequences that sit at the end of the list.
    sc.x1 = i == G - 1 ? W + 1 : x1;
    // The first sequence of the range (it may be empty, sitting at x0) and the
    // sequence of its last tile.
    if (!gd_find(p, sc.x0, true, sc.b0, sc.h0, sc.P0)) sc.b0 = p.B;
    if (!gd_find(p, x1 - 1, false, sc.bL, sc.hL, sc.PL)) {
        sc.bL = sc.b0;
        sc.hL = sc.h0;
        sc.PL = sc.P0;
    }
}

// Walks this CTA's units in order; every role warp runs its own copy.
struct GdIter {
    int un;         // fixed splits: next unit index
    int phase;      // balanced: 0 first sequence, 1 last, 2 those in between, 3 those after the last
    int b, h, tb;   // balanced: next sequence of phases 2 and 3, and its tile count
    long long P;    // balanced: its first tile in the list
};

__device__ __forceinline__ void gd_begin(const AttnParams &p, const GdSched &sc, GdIter &it) {
    it.un = blockIdx.x;
    it.phase = 0;
    it.b = it.h = it.tb = 0;
    it.P = 0;
}

// Steps (b, h, P) to the next sequence in (b, h) order.
__device__ __forceinline__ void gd_step(const AttnParams &p, int &b, int &h, long long &P, int &tb) {
    P += tb;
    if (++h >= p.Hkv) {
        h = 0;
        ++b;
        tb = b < p.B ? gd_tiles(p, b) : 0;
    }
}

// The piece of sequence (b, h), first tile Ps, that lies in this CTA's range.
__device__ __forceinline__ void gd_piece(const AttnParams &p, const GdSched &sc, int b, int h, long long Ps,
                                         GdUnit &u) {
    const int Ts = gd_tiles(p, b);
    const long long t0 = Ps < sc.x0 ? sc.x0 - Ps : 0;
    const long long t1 = Ps + Ts > sc.x1 ? sc.x1 - Ps : Ts;
    u.b = b;
    u.h_kv = h;
    u.L = imax(0, imin(p.seqlens[b], p.kv_cap));
    u.tile_begin = kv_window_lo(p, u.L) / 128 + static_cast<int>(t0);
    u.T = Ts > 0 ? static_cast<int>(t1 - t0) : 0;
    u.whole = t0 == 0 && t1 == Ts;
    if (Ts > 0) {
        const int first = gd_cta_of(Ps, sc.W, gridDim.x);
        u.slot = static_cast<int>(blockIdx.x) - first;
        u.n_pieces = gd_cta_of(Ps + Ts - 1, sc.W, gridDim.x) - first + 1;
    } else {
        u.slot = 0;
        u.n_pieces = 1;
    }
}

__device__ __forceinline__ bool gd_next(const AttnParams &p, const GdSched &sc, GdIter &it, GdUnit &u) {
    if (!sc.streamk) {
        if (it.un >= p.B * p.Hkv * p.num_splits) return false;
        const int idx = it.un;
        it.un += gridDim.x;
        const int split = idx % p.num_splits;
        const int rem = idx / p.num_splits;
        u.h_kv = rem % p.Hkv;
        u.b = rem / p.Hkv;
        u.L = imax(0, imin(p.seqlens[u.b], p.kv_cap));
        const int n_tiles = (u.L + 127) / 128;
        u.tile_begin = kv_window_lo(p, u.L) / 128 + split * p.split_tiles;
        u.T = imax(0, imin(u.tile_begin + p.split_tiles, n_tiles) - u.tile_begin);
        u.slot = split;
        u.n_pieces = p.num_splits;
        u.whole = p.num_splits == 1;
        return true;
    }
    if (sc.b0 >= p.B) return false;
    const bool last_differs = sc.bL != sc.b0 || sc.hL != sc.h0;
    if (it.phase == 0) {
        gd_piece(p, sc, sc.b0, sc.h0, sc.P0, u);
        it.phase = last_differs ? 1 : 3;
        it.b = sc.b0;
        it.h = sc.h0;
        it.P = sc.P0;
        it.tb = gd_tiles(p, sc.b0);
        gd_step(p, it.b, it.h, it.P, it.tb);
        return true;
    }
    if (it.phase == 1) {
        gd_piece(p, sc, sc.bL, sc.hL, sc.PL, u);
        it.phase = 2;
        return true;
    }
    if (it.phase == 2) {
        if (it.b != sc.bL || it.h != sc.hL) {
            gd_piece(p, sc, it.b, it.h, it.P, u);
            gd_step(p, it.b, it.h, it.P, it.tb);
            return true;
        }
        it.phase = 3;
        gd_step(p, it.b, it.h, it.P, it.tb);  // past the last sequence
    }
    if (it.b >= p.B || it.P >= sc.x1) return false;
    gd_piece(p, sc, it.b, it.h, it.P, u);
    gd_step(p, it.b, it.h, it.P, it.tb);
    return true;
}

}  // namespace qk4v8
