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

}  // namespace dbc
