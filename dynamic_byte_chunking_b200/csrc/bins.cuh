// Chunk and bin of one position (ByteFlow, paper.rainbus.top summary,
// "Method steps", stage 4; papernotes.org notes, "Key design 4"): the chunk of
// t is the last boundary s_c <= t; the bin is the offset inside the chunk
// (clamped to B-1), the fraction of the chunk, or the absolute position,
// depending on the mode.  Shared by the upsampling and its backward.
#pragma once

#include "common.cuh"

namespace dbc {

struct PosClass {
    int32_t chunk;   // global chunk row (idx_offsets[r] + c)
    int32_t bin;
};

__device__ __forceinline__ PosClass classify_position(int64_t p, const int64_t *offsets, int64_t T,
                                                      const int64_t *__restrict__ idx,
                                                      const int64_t *__restrict__ idx_offsets, int64_t rows,
                                                      int nbins, int mode, int32_t *st) {
    const int64_t r = offsets ? find_row(offsets, rows, p) : p / T;
    int64_t a, n;
    row_bounds(offsets, r, T, a, n);
    const int64_t t = p - a;
    const int64_t ia = idx_offsets[r];
    const int64_t kr = idx_offsets[r + 1] - ia;
    int64_t c = 0;
    if (kr <= 0 || idx[ia] != 0) {
        flag(st, DBC_ERR_BOUNDS);
    } else {
        int64_t lo = 0, hi = kr;     // idx[ia+lo] <= t < idx[ia+hi] (hi = kr: +inf)
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if (idx[ia + mid] <= t) lo = mid; else hi = mid;
        }
        c = lo;
    }
    const int64_t sc = kr > 0 ? idx[ia + c] : 0;
    int64_t b;
    if (mode == DBC_BIN_IN_CHUNK_OFFSET) {
        b = t - sc;
        if (b > nbins - 1) b = nbins - 1;
    } else if (mode == DBC_BIN_IN_CHUNK_FRACTION) {
        const int64_t nxt = (c + 1 < kr) ? idx[ia + c + 1] : n;
        const int64_t len = nxt - sc;
        b = len > 0 ? ((int64_t)nbins * (t - sc)) / len : 0;
    } else {
        b = ((int64_t)t * nbins) / n;
    }
    if (b < 0 || b >= nbins) {
        flag(st, DBC_ERR_BOUNDS);
        b = b < 0 ? 0 : nbins - 1;
    }
    return PosClass{(int32_t)(ia + c), (int32_t)b};
}

// The same classification for the 32 consecutive positions p0 .. p0 + 31 of one warp (lane i
// takes p0 + i; all lanes call it with the same p0).  When the 32 positions lie in one row whose
// boundary list starts at 0, the warp finds the chunk of p0 with a 33-way search (32 probes per
// round, three rounds for 2048 boundaries) instead of a binary search per lane, then reads the next
// 32 boundaries at once: each lane's chunk is the chunk of p0 plus the boundaries at or before it,
// counted from one 32-bit mask of boundary offsets.  Otherwise (a row break, an empty or malformed
// row) every lane takes classify_position.  Lanes past N return chunk -1.
__device__ __forceinline__ PosClass classify_warp(int64_t p0, int64_t N, const int64_t *offsets, int64_t T,
                                                  const int64_t *__restrict__ idx,
                                                  const int64_t *__restrict__ idx_offsets, int64_t rows,
                                                  int nbins, int mode, int32_t *st) {
    const int lane = threadIdx.x & 31;
    const int64_t p = p0 + lane;
    const int64_t pl = p0 + 31 < N ? p0 + 31 : N - 1;         // last position of the warp
    const int64_t r = offsets ? find_row(offsets, rows, p0) : p0 / T;
    int64_t a, n;
    row_bounds(offsets, r, T, a, n);
    const int64_t ia = idx_offsets[r];
    const int64_t kr = idx_offsets[r + 1] - ia;
    const bool fast = pl < a + n && kr > 0 && idx[ia] == 0;   // warp-uniform
    if (!fast) {
        if (p >= N) return PosClass{-1, 0};
        return classify_position(p, offsets, T, idx, idx_offsets, rows, nbins, mode, st);
    }
    const int64_t t0 = p0 - a, t = p - a;
    // chunk of t0: idx[ia + lo] <= t0 < idx[ia + hi] (hi == kr: +inf).  Each round probes 32
    // boundaries strictly inside (lo, hi), non-decreasing with the lane; those at or before t0 are
    // a prefix of the lanes, so the last of them is the new lo and the next probe the new hi.
    int64_t lo = 0, hi = kr;
    while (hi - lo > 1) {
        const int64_t probe = lo + 1 + ((hi - lo - 1) * lane) / 32;
        const unsigned m = __ballot_sync(0xffffffffu, idx[ia + probe] <= t0);
        const int cnt = __popc(m);
        const int64_t nlo = cnt ? __shfl_sync(0xffffffffu, probe, cnt - 1) : lo;
        const int64_t nhi = __shfl_sync(0xffffffffu, probe, cnt < 32 ? cnt : 31);
        lo = nlo;
        if (cnt < 32) hi = nhi;
    }
    const int64_t c0 = lo;
    // boundary offsets after t0 within the warp's 32 positions
    const int64_t jb = c0 + 1 + lane;
    const int64_t bj = jb < kr ? idx[ia + jb] : INT64_MAX;
    const int64_t off = bj - t0;
    const unsigned M = __reduce_or_sync(0xffffffffu, (off >= 1 && off < 32) ? (1u << off) : 0u);
    if (p >= N) return PosClass{-1, 0};
    const unsigned upto = M & ((2u << lane) - 1u);            // boundaries at offsets 1 .. lane
    const int64_t c = c0 + __popc(upto);
    const int64_t sc = upto ? t0 + (31 - __clz(upto)) : idx[ia + c0];
    int64_t b;
    if (mode == DBC_BIN_IN_CHUNK_OFFSET) {
        b = t - sc;
        if (b > nbins - 1) b = nbins - 1;
    } else if (mode == DBC_BIN_IN_CHUNK_FRACTION) {
        const int64_t nxt = (c + 1 < kr) ? idx[ia + c + 1] : n;
        const int64_t len = nxt - sc;
        b = len > 0 ? ((int64_t)nbins * (t - sc)) / len : 0;
    } else {
        b = ((int64_t)t * nbins) / n;
    }
    if (b < 0 || b >= nbins) {
        flag(st, DBC_ERR_BOUNDS);
        b = b < 0 ? 0 : nbins - 1;
    }
    return PosClass{(int32_t)(ia + c), (int32_t)b};
}

}  // namespace dbc
