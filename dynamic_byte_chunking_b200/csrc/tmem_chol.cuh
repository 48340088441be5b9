// Blocked Cholesky of (I + S) held entirely in tensor memory (d = 256).
//
// A 256 x 256 fp32 matrix fills one SM's TMEM: rows 0..127 sit in lanes
// 0..127 at columns [0, 256), rows 128..255 in the same lanes at columns
// [256, 512).  256 threads: thread (warp w, lane l) owns row
// (w/4)*128 + (w%4)*32 + l, the lanes its warp may address.  The identity is
// implicit: the stored diagonal is the excess e, the factor's diagonal is
// sqrt(1 + e).
//
// Per 64-column panel: every thread loads its row's 64 panel entries with
// tcgen05.ld, the panel is factored in registers in 16-column sub-panels
// (diagonal block by shuffles, then a solve and a rank-16 update per row:
// two barriers per sub-panel),
// the panel rows are split into three bf16 pieces (hi + mid + lo carries the
// fp32 value) and staged in shared memory, and the trailing columns are
// updated in place by tcgen05 MMAs with negated A over the six piece
// products whose sum is accurate to fp32 (hi.hi, hi.mid, mid.hi, hi.lo,
// lo.hi, mid.mid).  Two uses:
//
//  * FACTOR (segment start state M_s = I + P_s): the upper triangle, which
//    starts at zero, carries B = L^{-T} along (row i of the identity solved
//    against the factor, B_ii = 1 / L_ii), so one sweep yields both; the
//    panels of B are saved and A = B B^T = M_s^{-1} is formed at the end on
//    tcgen05 and stored as three bf16 pieces.
//  * INSEG (one segment): G' = X (c V)^T is accumulated straight into TMEM
//    (V = X_s A_s in pieces), factored in place, and the excess of each
//    column gives dR_t = log1p(e_t) / 2.
#pragma once

#include "tc.cuh"

namespace dbc {
namespace cr {

struct TmemChol {
    static constexpr int NT = 256;
    static constexpr uint32_t XT = 128 * 128;             // 128-row x 64-K bf16 tile
    static constexpr uint32_t PIECE = 256 * 128;          // 256-row x 64-K bf16 tile
    static constexpr uint32_t PANEL = 3 * PIECE;          // staged panel (three pieces)
    static constexpr uint32_t GSTAGE = 2 * XT + PIECE;    // G' GEMM stage: X (two row blocks) + V piece
    static constexpr uint32_t REGION = (2 * GSTAGE > PANEL) ? 2 * GSTAGE : PANEL;
    static constexpr uint32_t DONE = 256 * 65 * 4;           // finished panel values [256][65] fp32
    static constexpr size_t SMEM = REGION + DONE + 1024;
};

// Rank-16 update and shift of the live panel columns of one row:
// v[p] <- v[16 + p] - sum_c a[c] L[kb+16+p][kb+c] for p in [0, P), with the
// solved sub-panel stored column-major in shared memory (sLT[c * 64 + p]).
// The loop runs column-outer so the P updates of one step are independent.
// Entries p >= zfrom are set to zero instead: the part right of the diagonal
// of a panel row in the L role, which in the factor mode carries B and is
// still zero there.
template <int P>
__device__ __forceinline__ void rank16_shift(float (&v)[64], const float (&a)[16], const float *sLT, int zfrom) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const float4 *lr = reinterpret_cast<const float4 *>(sLT + c * 64);
#pragma unroll
        for (int p4 = 0; p4 < P / 4; ++p4) {
            const float4 l = lr[p4];
            v[16 + 4 * p4 + 0] = fmaf(-a[c], l.x, v[16 + 4 * p4 + 0]);
            v[16 + 4 * p4 + 1] = fmaf(-a[c], l.y, v[16 + 4 * p4 + 1]);
            v[16 + 4 * p4 + 2] = fmaf(-a[c], l.z, v[16 + 4 * p4 + 2]);
            v[16 + 4 * p4 + 3] = fmaf(-a[c], l.w, v[16 + 4 * p4 + 3]);
        }
    }
#pragma unroll
    for (int p = 0; p < P; ++p) v[p] = p >= zfrom ? 0.f : v[16 + p];
}

// Six piece products of a three-way split (dropped terms are below 2^-24):
// hi.hi, hi.mid, mid.hi, hi.lo, lo.hi, mid.mid.
__device__ __forceinline__ constexpr int pair_a(int i) { return i == 2 ? 1 : (i == 4 ? 2 : (i == 5 ? 1 : 0)); }
__device__ __forceinline__ constexpr int pair_b(int i) { return i == 1 ? 1 : (i == 3 ? 2 : (i == 5 ? 1 : 0)); }

__device__ __forceinline__ void split3v(float v, uint16_t &h, uint16_t &m, uint16_t &l) {
    const __nv_bfloat16 bh = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(bh);
    const __nv_bfloat16 bm = __float2bfloat16_rn(r1);
    const __nv_bfloat16 bl = __float2bfloat16_rn(r1 - __bfloat162float(bm));
    h = __bfloat16_as_ushort(bh);
    m = __bfloat16_as_ushort(bm);
    l = __bfloat16_as_ushort(bl);
}

// Stages 64 values of one row as three K-major pieces (row `row` of each
// 256-row tile) and, when gdst != nullptr, also writes them to global
// pieces gdst[p * pstride + k] (row-major bf16).
__device__ __forceinline__ void stage_row(uint32_t region, int row, const float (&a)[64], __nv_bfloat16 *gdst,
                                          size_t pstride) {
#pragma unroll
    for (int k8 = 0; k8 < 8; ++k8) {
        uint32_t hh[4], mm[4], ll[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint16_t h0, m0, l0, h1, m1, l1;
            split3v(a[k8 * 8 + 2 * q], h0, m0, l0);
            split3v(a[k8 * 8 + 2 * q + 1], h1, m1, l1);
            hh[q] = (uint32_t)h0 | ((uint32_t)h1 << 16);
            mm[q] = (uint32_t)m0 | ((uint32_t)m1 << 16);
            ll[q] = (uint32_t)l0 | ((uint32_t)l1 << 16);
        }
        const uint32_t off = tc::kmajor_off(row, k8 * 8);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(region + off), "r"(hh[0]), "r"(hh[1]),
                     "r"(hh[2]), "r"(hh[3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(region + TmemChol::PIECE + off), "r"(mm[0]),
                     "r"(mm[1]), "r"(mm[2]), "r"(mm[3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(region + 2 * TmemChol::PIECE + off),
                     "r"(ll[0]), "r"(ll[1]), "r"(ll[2]), "r"(ll[3])
                     : "memory");
        if (gdst) {
            *reinterpret_cast<uint4 *>(gdst + k8 * 8) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
            *reinterpret_cast<uint4 *>(gdst + pstride + k8 * 8) = make_uint4(mm[0], mm[1], mm[2], mm[3]);
            *reinterpret_cast<uint4 *>(gdst + 2 * pstride + k8 * 8) = make_uint4(ll[0], ll[1], ll[2], ll[3]);
        }
    }
}

// D[block b rows, columns c0 .. c0+N) (+/-)= sum of the six piece products of
// A (rows a_row0 .. +128 of the staged tiles) and B (rows b_row0 .. +N).
__device__ __forceinline__ void issue_split_mma(uint32_t d_tmem, uint32_t region_a, uint32_t region_b,
                                                int a_row0, int b_row0, uint32_t idesc, bool first) {
#pragma unroll
    for (int pr = 0; pr < 6; ++pr) {
        const uint32_t pa = region_a + (uint32_t)pair_a(pr) * TmemChol::PIECE + (uint32_t)a_row0 * 128;
        const uint32_t pb = region_b + (uint32_t)pair_b(pr) * TmemChol::PIECE + (uint32_t)b_row0 * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(d_tmem, tc::sdesc(pa + kk * 32, 16, 1024), tc::sdesc(pb + kk * 32, 16, 1024), idesc,
                         (first && pr == 0 && kk == 0) ? 0u : 1u);
    }
}

// Runtime N of the negated trailing update (N = 256 - j1, a multiple of 64).
__device__ __forceinline__ uint32_t idesc_neg(int N) { return tc::idesc_bf16(128, N, false, false, true); }

template <bool FACTOR>
__global__ void __launch_bounds__(TmemChol::NT, 1) tmem_chol_kernel(
    const __nv_bfloat16 *__restrict__ H, Segs S, const float *__restrict__ Pbuf, __nv_bfloat16 *Bscr,
    __nv_bfloat16 *A3, const __nv_bfloat16 *__restrict__ V3, int64_t N, float *dR, int32_t *st) {
    constexpr int D = 256;
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[2];
    __shared__ uint32_t tmem_base;
    __shared__ __align__(16) float s_LT[16][64];    // solved sub-panel of the panel's rows, column-major
    __shared__ __align__(16) float s_LdT[16][16];   // factored 16 x 16 diagonal block, column-major
    __shared__ __align__(16) float s_rl[16];        // 1 / L_kk of the diagonal block
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int blk = warp >> 2, lb = (warp & 3) * 32;
    const int row = blk * 128 + lb + lane;
    const uint32_t region = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    float *done = reinterpret_cast<float *>(smraw + (region - tc::smem_u32(smraw)) + TmemChol::REGION);
    for (int e = tid; e < 16 * 64; e += TmemChol::NT) (&s_LT[0][0])[e] = 0.f;
    if (warp == 0) tc::tmem_alloc(&tmem_base, 512);
    if (tid == 0) {
        tc::mbar_init(&mbar[0], 1);
        tc::mbar_init(&mbar[1], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const uint32_t trow = tbase + ((uint32_t)lb << 16) + (uint32_t)(blk * 256);
    uint32_t ph0 = 0, ph1 = 0;      // mbarrier phases (uniform across threads)
    bool ok = true;
    const int nseg = *S.nseg;

    for (int s = blockIdx.x; s < nseg && ok; s += gridDim.x) {
        const int len = S.len[s];
        const int64_t start = S.start[s];
        const int n = FACTOR ? D : len;

        // ---------------- load the matrix into TMEM
        if (FACTOR) {
            const float *P = Pbuf + (size_t)s * D * D;            // c-scaled prefix Gram
            float *stg = reinterpret_cast<float *>(smraw + (region - tc::smem_u32(smraw)));
            for (int q = 0; q < D / 64; ++q) {
                for (int e = tid; e < D * 16; e += TmemChol::NT) {           // 256 rows x 16 float4
                    const int r = e >> 4, c4 = e & 15;
                    const float4 x = *reinterpret_cast<const float4 *>(P + (size_t)r * D + q * 64 + c4 * 4);
                    float *d = stg + r * 65 + c4 * 4;
                    d[0] = x.x; d[1] = x.y; d[2] = x.z; d[3] = x.w;
                }
                __syncthreads();
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int col = q * 64 + j * 16 + i;
                        v[i] = col <= row ? stg[row * 65 + j * 16 + i] : 0.f;
                    }
                    tc::tmem_st16(trow + (uint32_t)(q * 64 + j * 16), v);
                }
                __syncthreads();
            }
            tc::tmem_wait_st();
        } else {
            // G' = X (c V)^T over 3 pieces x (D/64) feature chunks, two stages
            const __nv_bfloat16 *X = H + start * D;
            constexpr int KC = D / 64, NCH = 3 * KC;
            auto load = [&](int c, uint32_t sb) {
                const int p = c / KC, kc = c % KC;
                for (int e = tid; e < 256 * 8; e += TmemChol::NT) {
                    const int r = e >> 3, ch = e & 7;
                    const bool in = r < len;
                    const __nv_bfloat16 *gx = X + (size_t)(in ? r : 0) * D + kc * 64 + ch * 8;
                    const uint32_t xo = (r < 128) ? tc::kmajor_off(r, ch * 8) : TmemChol::XT + tc::kmajor_off(r - 128, ch * 8);
                    tc::cp_async16(sb + xo, gx, in ? 16u : 0u);
                    const __nv_bfloat16 *gv = V3 + (size_t)p * N * D + (size_t)(start + (in ? r : 0)) * D + kc * 64 + ch * 8;
                    tc::cp_async16(sb + 2 * TmemChol::XT + tc::kmajor_off(r, ch * 8), gv, in ? 16u : 0u);
                }
            };
            constexpr uint32_t idg = tc::idesc_bf16(128, 256, false, false);
            load(0, region);
            tc::cp_async_commit();
            for (int c = 0; c < NCH; ++c) {
                if (c + 1 < NCH) {
                    if (c >= 1) {     // stage (c+1)%2 was read by the MMAs of chunk c-1
                        ok &= tc::mbar_wait(&mbar[(c + 1) & 1], ((c + 1) & 1) ? ph1 : ph0, st);
                        if ((c + 1) & 1) ph1 ^= 1; else ph0 ^= 1;
                    }
                    load(c + 1, region + (uint32_t)((c + 1) & 1) * TmemChol::GSTAGE);
                }
                tc::cp_async_commit();
                tc::cp_async_wait<1>();
                tc::fence_async_smem();
                __syncthreads();
                if (tid == 0) {
                    tc::fence_after_sync();
                    const uint32_t sb = region + (uint32_t)(c & 1) * TmemChol::GSTAGE;
#pragma unroll
                    for (int b = 0; b < 2; ++b)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma_bf16(tbase + (uint32_t)(b * 256), tc::sdesc(sb + b * TmemChol::XT + kk * 32, 16, 1024),
                                         tc::sdesc(sb + 2 * TmemChol::XT + kk * 32, 16, 1024), idg,
                                         (c > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&mbar[c & 1]);
                }
                __syncthreads();
            }
            // wait for the last two chunks' MMAs
            for (int c = (NCH >= 2 ? NCH - 2 : 0); c < NCH; ++c) {
                ok &= tc::mbar_wait(&mbar[c & 1], (c & 1) ? ph1 : ph0, st);
                if (c & 1) ph1 ^= 1; else ph0 ^= 1;
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;

        // ---------------- panels
        __nv_bfloat16 *Bs = FACTOR ? Bscr + (size_t)s * 3 * D * D : nullptr;
        for (int j0 = 0; j0 < n; j0 += 64) {
            const int nb = min(64, n - j0);
            const int j1 = j0 + nb;
            float v[64];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float t16[16];
                tc::tmem_ld16(trow + (uint32_t)(j0 + j * 16), t16);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[j * 16 + i] = t16[i];
            }
            if (FACTOR && row >= j0 && row < j1) {
                // this row's B entries right of its diagonal start from zero: B_im = 0 for m < i,
                // so nothing before this panel contributes to them
#pragma unroll
                for (int k = 0; k < 64; ++k)
                    if (j0 + k > row) v[k] = 0.f;
            }
            // ---- factor the panel in 16-column sub-panels: (1) the 16 x 16 diagonal block by its
            // half-warp with shuffles, (2) every other live row solves its 16 values against it,
            // (3) rank-16 update of the later panel columns with a shift by 16, so the current
            // sub-panel is always v[0..15].  Two barriers per sub-panel.
            const int rel = row - j0;
            const int nsub = (nb + 15) / 16;
#pragma unroll 1
            for (int q = 0; q < nsub; ++q) {
                const int kb = 16 * q;
                const int ii = rel - kb;
                const bool diag = ii >= 0 && ii < 16;
                float a[16];
                if (diag) {
                    // branch-free (selects only): the half-warp stays converged for its shuffles,
                    // and the per-pivot work on the serial path is one broadcast, one rsqrt and
                    // one fma; each lane keeps its own pivot's values and writes them afterwards
                    const int lb0 = lane & 16;
                    const unsigned mask = 0xFFFFu << lb0;
                    float rl_mine = 1.f, e_mine = 0.f;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float e = __shfl_sync(mask, v[c], lb0 + c);   // excess of column c
                        const float rlc = rsqrtf(1.f + e);
                        const float li = v[c] * rlc;                        // L_ii,c for ii > c
#pragma unroll
                        for (int c2 = 0; c2 < 16; ++c2) {
                            if (c2 > c) {
                                const float w = __shfl_sync(mask, v[c], lb0 + c2);
                                const float u = fmaf(-li, w * rlc, v[c2]);
                                v[c2] = ii >= c2 ? u : v[c2];
                            }
                        }
                        const bool piv = ii == c;
                        v[c] = piv ? (1.f + e) * rlc : (ii > c ? li : v[c]);  // L_cc on the pivot row
                        rl_mine = piv ? rlc : rl_mine;
                        e_mine = piv ? e : e_mine;
                    }
                    s_rl[ii] = rl_mine;
                    if (!FACTOR && kb + ii < nb) dR[start + j0 + kb + ii] = 0.5f * log1pf(e_mine);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float x = c <= ii ? v[c] : 0.f;
                        s_LdT[c][ii] = x;
                        if (c <= ii) done[row * 65 + kb + c] = x;
                    }
                }
                __syncthreads();
                const bool live = FACTOR || ii >= 16;        // INSEG rows at or above the block are done
                if (live) {
                    // right-looking solve against the diagonal block: a[m] is final once the
                    // columns before m are applied; a diagonal-block row takes the B role
                    // (B_im = 0 for m < ii, B_ii = 1/L_ii)
                    float rl[16];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float4 r4 = reinterpret_cast<const float4 *>(s_rl)[j];
                        rl[4 * j] = r4.x; rl[4 * j + 1] = r4.y; rl[4 * j + 2] = r4.z; rl[4 * j + 3] = r4.w;
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        float am = v[m] * rl[m];
                        if (diag && m <= ii) am = m == ii ? rl[m] : 0.f;
                        a[m] = am;
                        const float4 *lr = reinterpret_cast<const float4 *>(&s_LdT[m][0]);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if (4 * j + 3 > m) {
                                const float4 l = lr[j];
                                if (4 * j + 0 > m) v[4 * j + 0] = fmaf(-am, l.x, v[4 * j + 0]);
                                if (4 * j + 1 > m) v[4 * j + 1] = fmaf(-am, l.y, v[4 * j + 1]);
                                if (4 * j + 2 > m) v[4 * j + 2] = fmaf(-am, l.z, v[4 * j + 2]);
                                v[4 * j + 3] = fmaf(-am, l.w, v[4 * j + 3]);
                            }
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (!(diag && c <= ii)) done[row * 65 + kb + c] = a[c];
                    if (ii >= 16 && rel < 64) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) s_LT[c][rel] = a[c];
                    }
                }
                __syncthreads();
                if (live && q + 1 < nsub) {
                    const float *sLT = &s_LT[0][kb + 16];
                    const int zfrom = (FACTOR && ii >= 16 && rel < 64) ? ii - 15 : 64;
                    if (q == 0) rank16_shift<48>(v, a, sLT, zfrom);
                    else if (q == 1) rank16_shift<32>(v, a, sLT, zfrom);
                    else rank16_shift<16>(v, a, sLT, zfrom);
                }
            }
#pragma unroll
            for (int k = 0; k < 64; ++k) v[k] = k < nb ? done[row * 65 + k] : 0.f;
            // operand rows: FACTOR rows < j1 carry B (0 below the diagonal, 1/L_ii on it),
            // INSEG rows < j1 are not updated (zero); rows >= j1 carry L.
            if (row < j1) {
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    const int col = j0 + k;
                    v[k] = !FACTOR ? 0.f : (col < row ? 0.f : (col == row ? 1.f / v[k] : v[k]));
                }
            } else {
#pragma unroll
                for (int k = 0; k < 64; ++k)
                    if (k >= nb) v[k] = 0.f;
            }
            if (FACTOR) {
                // B panel -> global (rows >= j1 are zero in these columns and are never stored: the
                // product B B^T below zero-fills them); operand rows -> smem
                stage_row(region, row, v, row < j1 ? Bs + (size_t)row * D + j0 : nullptr, (size_t)D * D);
            } else if (j1 < n) {
                stage_row(region, row, v, nullptr, 0);
            }
            if (FACTOR && j1 < n && row >= j0 && row < j1) {
                // the trailing updates of earlier panels reached this row's upper part while it was an
                // L row; its B entries right of the panel start from zero (warps of the diagonal block)
                float z[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) z[i] = 0.f;
                for (int c0 = j1; c0 < D; c0 += 16) tc::tmem_st16(trow + (uint32_t)c0, z);
                tc::tmem_wait_st();
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            __syncthreads();
            if (j1 < n) {
                if (tid == 0) {
                    tc::fence_after_sync();
                    const uint32_t idn = idesc_neg(256 - j1);
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        if (!FACTOR && (b + 1) * 128 <= j1) continue;
                        issue_split_mma(tbase + (uint32_t)(b * 256 + j1), region, region, b * 128, j1, idn, false);
                    }
                    tc::mma_commit(&mbar[0]);
                }
                ok &= tc::mbar_wait(&mbar[0], ph0, st);
                ph0 ^= 1;
                tc::fence_after_sync();
                ok = __syncthreads_and(ok) != 0;
                if (!ok) break;
            } else {
                tc::fence_before_sync();
                __syncthreads();
                tc::fence_after_sync();
            }
        }
        if (!ok) break;

        // ---------------- FACTOR: A = B B^T from the saved panels, split into pieces
        if (FACTOR) {
            for (int q = 0; q < D / 64; ++q) {
                for (int e = tid; e < 3 * 256 * 8; e += TmemChol::NT) {
                    const int p = e / 2048, r = (e >> 3) & 255, ch = e & 7;
                    const bool nz = r < q * 64 + 64;        // B rows beyond are zero in these columns
                    const __nv_bfloat16 *gsrc = Bs + (size_t)p * D * D + (size_t)(nz ? r : 0) * D + q * 64 + ch * 8;
                    tc::cp_async16(region + (uint32_t)p * TmemChol::PIECE + tc::kmajor_off(r, ch * 8), gsrc,
                                   nz ? 16u : 0u);
                }
                tc::cp_async_commit();
                tc::cp_async_wait<0>();
                tc::fence_async_smem();
                __syncthreads();
                if (tid == 0) {
                    tc::fence_after_sync();
                    constexpr uint32_t idp = tc::idesc_bf16(128, 256, false, false);
                    for (int b = 0; b < 2; ++b) {
                        if (b == 1 && q < 2) continue;          // rows 128.. of B vanish in columns < 128
                        issue_split_mma(tbase + (uint32_t)(b * 256), region, region, b * 128, 0, idp,
                                        b == 0 ? (q == 0) : (q == 2));
                    }
                    tc::mma_commit(&mbar[0]);
                }
                ok &= tc::mbar_wait(&mbar[0], ph0, st);
                ph0 ^= 1;
                tc::fence_after_sync();
                ok = __syncthreads_and(ok) != 0;
                if (!ok) break;
            }
            if (!ok) break;
            // A -> three bf16 pieces, staged per 64-column block in shared memory (row-major, 144-byte
            // rows) and written out as whole 128-byte row segments
            __nv_bfloat16 *Ag = A3 + (size_t)s * 3 * D * D;
            uint8_t *stg = smraw + (region - tc::smem_u32(smraw));
            constexpr int RS = 144;
#pragma unroll 1
            for (int cb = 0; cb < D; cb += 64) {
#pragma unroll 1
                for (int j = 0; j < 4; ++j) {
                    float t16[16];
                    tc::tmem_ld16(trow + (uint32_t)(cb + 16 * j), t16);
                    uint32_t hh[8], mm[8], ll[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint16_t h0, m0, l0, h1, m1, l1;
                        split3v(t16[2 * q], h0, m0, l0);
                        split3v(t16[2 * q + 1], h1, m1, l1);
                        hh[q] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                        mm[q] = (uint32_t)m0 | ((uint32_t)m1 << 16);
                        ll[q] = (uint32_t)l0 | ((uint32_t)l1 << 16);
                    }
                    uint4 *d0 = reinterpret_cast<uint4 *>(stg + (size_t)row * RS + j * 32);
                    uint4 *d1 = reinterpret_cast<uint4 *>(stg + (size_t)(256 + row) * RS + j * 32);
                    uint4 *d2 = reinterpret_cast<uint4 *>(stg + (size_t)(512 + row) * RS + j * 32);
                    d0[0] = make_uint4(hh[0], hh[1], hh[2], hh[3]); d0[1] = make_uint4(hh[4], hh[5], hh[6], hh[7]);
                    d1[0] = make_uint4(mm[0], mm[1], mm[2], mm[3]); d1[1] = make_uint4(mm[4], mm[5], mm[6], mm[7]);
                    d2[0] = make_uint4(ll[0], ll[1], ll[2], ll[3]); d2[1] = make_uint4(ll[4], ll[5], ll[6], ll[7]);
                }
                __syncthreads();
                for (int e = tid; e < 3 * 256 * 8; e += TmemChol::NT) {
                    const int pr = e >> 3, ch = e & 7;                 // piece-row (piece * 256 + row), chunk
                    const uint4 x = *reinterpret_cast<const uint4 *>(stg + (size_t)pr * RS + ch * 16);
                    const int pc = pr >> 8, r = pr & 255;
                    *reinterpret_cast<uint4 *>(Ag + (size_t)pc * D * D + (size_t)r * D + cb + ch * 8) = x;
                }
                __syncthreads();
            }
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

}  // namespace cr
}  // namespace dbc
