// Right-looking panel Cholesky of (I + A) with the identity kept implicit.
//
// A is the lower part of an nrows x ncols row-major block in global memory
// (nrows >= ncols; rows >= ncols are extra rows appended below the square
// part, which receive the solve X L^{-T} of the square factor).  Only the
// first ncols columns are factored.  When a column is reached, its stored
// diagonal holds the Schur complement minus one -- the "excess" e -- so the
// factor's diagonal is sqrt(1 + e) and the 1 is never rounded into large
// entries.  Used twice by the coding-rate path:
//   * per segment start, on [P_s ; I]: the bottom block becomes L_s^{-T};
//   * per segment, on the in-segment Gram G': e_t gives dR_t = log1p(e_t)/2.
//
// One CTA, NT threads.  Panels of PW columns: thread t holds panel row
// (j0 + t) in registers while the panel is factored (two barriers per
// column), then the panel is staged transposed in shared memory and the
// trailing lower region is updated in 128 x (NT/4) register tiles of 4 x 8
// per thread straight in global memory.
#pragma once

#include "common.cuh"

namespace dbc {
namespace pc {

template <int PW, int NT>
struct PanelChol {
    static constexpr int TN = NT / 4;                 // trailing tile width
    static constexpr int NTP = NT + (TN > 128 ? TN : 128);   // staged row stride (zero padded)
    static constexpr size_t SMEM = (size_t)PW * NTP * sizeof(float) + (NT + 64) * sizeof(float);
};

// bottom_identity: rows >= ncols started as the identity (row ncols+i is
// e_i), so in panel [j0, j0+PW) rows ncols+i with i >= j0+PW are still zero
// and their trailing tiles are skipped.
template <int PW, int NT>
__device__ __forceinline__ void panel_chol(float *A, int ld, int nrows, int ncols, bool bottom_identity,
                                           float *dR, bool write_back_bottom, float *sm) {
    using C = PanelChol<PW, NT>;
    constexpr int NTP = C::NTP, TN = C::TN;
    float *PsT = sm;                    // [PW][NTP]: panel transposed, zero beyond the panel rows
    float *s_col = sm + PW * NTP;       // [NT]
    float *s_e = s_col + NT;            // [1]
    const int t = threadIdx.x;
    for (int e = t; e < PW * NTP; e += NT) PsT[e] = 0.f;
    __syncthreads();
    for (int j0 = 0; j0 < ncols; j0 += PW) {
        const int nb = min(PW, ncols - j0);
        const int m = nrows - j0;
        float r[PW];
        const bool have = t < m;
        const float *src = A + (size_t)(j0 + t) * ld + j0;
#pragma unroll
        for (int k = 0; k < PW; ++k) r[k] = (have && k < nb) ? src[k] : 0.f;
#pragma unroll
        for (int k = 0; k < PW; ++k) {
            if (k < nb) {
                if (t == k) *s_e = r[k];
                __syncthreads();
                const float e = *s_e;
                const float l = sqrtf(1.f + e);
                if (t == k) {
                    r[k] = l;
                    if (dR) dR[j0 + k] = 0.5f * log1pf(e);
                } else if (t > k && have) {
                    r[k] = r[k] / l;
                }
                s_col[t] = r[k];
                __syncthreads();
                if (t > k && have) {
                    const float a = r[k];
#pragma unroll
                    for (int p = k + 1; p < PW; ++p) r[p] = fmaf(-a, s_col[p], r[p]);
                }
            }
        }
        // stage the panel for the trailing update; keep the appended rows' solve
#pragma unroll
        for (int k = 0; k < PW; ++k) PsT[k * NTP + t] = have ? r[k] : 0.f;
        if (write_back_bottom && have && j0 + t >= ncols) {
            float *dst = A + (size_t)(j0 + t) * ld + j0;
#pragma unroll
            for (int k = 0; k < PW; ++k)
                if (k < nb) dst[k] = r[k];
        }
        __syncthreads();
        const int j1 = j0 + nb;
        if (j1 < ncols) {
            const int ty = t / (NT / 32), tx = t % (NT / 32);     // 32 x (NT/32) threads
            const int rows_tr = nrows - j1, cols_tr = ncols - j1;
            const int TI = (rows_tr + 127) / 128, TJ = (cols_tr + TN - 1) / TN;
            for (int I = 0; I < TI; ++I) {
                const int row0 = j1 + I * 128;
                if (bottom_identity && row0 >= ncols && row0 - ncols >= j1) break;   // rows still zero
                for (int J = 0; J < TJ; ++J) {
                    const int col0 = j1 + J * TN;
                    if (col0 > row0 + 127 && row0 + 127 < ncols) break;               // above the diagonal
                    float acc[4][8];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
#pragma unroll
                        for (int c = 0; c < 8; ++c) acc[q][c] = 0.f;
                    const int ra = row0 - j0 + ty * 4;        // staged column of this thread's rows
                    const int ca = col0 - j0 + tx * 8;
#pragma unroll 4
                    for (int k = 0; k < nb; ++k) {
                        const float *pk = PsT + k * NTP;
                        const float4 a4 = *reinterpret_cast<const float4 *>(pk + ra);
                        const float4 b0 = *reinterpret_cast<const float4 *>(pk + ca);
                        const float4 b1 = *reinterpret_cast<const float4 *>(pk + ca + 4);
                        const float a[4] = {a4.x, a4.y, a4.z, a4.w};
                        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int c = 0; c < 8; ++c) acc[q][c] = fmaf(a[q], b[c], acc[q][c]);
                    }
                    const int p0 = col0 + tx * 8;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int i = row0 + ty * 4 + q;
                        if (i >= nrows) continue;
                        float *rowp = A + (size_t)i * ld + p0;
                        if (p0 + 7 < ncols && (i >= ncols || p0 + 7 <= i)) {
                            float4 *v = reinterpret_cast<float4 *>(rowp);
                            float4 x0 = v[0], x1 = v[1];
                            x0.x -= acc[q][0]; x0.y -= acc[q][1]; x0.z -= acc[q][2]; x0.w -= acc[q][3];
                            x1.x -= acc[q][4]; x1.y -= acc[q][5]; x1.z -= acc[q][6]; x1.w -= acc[q][7];
                            v[0] = x0;
                            v[1] = x1;
                        } else {
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                const int p = p0 + c;
                                if (p < ncols && (i >= ncols || p <= i)) rowp[c] -= acc[q][c];
                            }
                        }
                    }
                }
            }
        }
        __syncthreads();
    }
}

}  // namespace pc
}  // namespace dbc
