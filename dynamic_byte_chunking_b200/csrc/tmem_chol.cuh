// Blocked Cholesky of (I + S) held entirely in tensor memory (d = 256).
//
// A 256 x 256 fp32 matrix fills one SM's TMEM: rows 0..127 sit in lanes
// 0..127 at columns [0, 256), rows 128..255 in the same lanes at columns
// [256, 512).  256 threads: thread (warp w, lane l) owns row
// (w/4)*128 + (w%4)*32 + l, the lanes its warp may address.  The identity is
// implicit: the stored diagonal is the excess e, the factor's diagonal is
// sqrt(1 + e).
//
// Per 16-column panel: every thread loads its row's 16 panel entries with
// tcgen05.ld; the 16 x 16 diagonal block is factored by its half-warp with
// shuffles, every other row solves its 16 values against it, the values are
// split into three bf16 pieces (hi + mid + lo carries the fp32 value) and
// staged in shared memory, and all later columns are updated in place by
// tcgen05 MMAs with negated A over the six piece products whose sum is
// accurate to fp32 (hi.hi, hi.mid, mid.hi, hi.lo, lo.hi, mid.mid), K = 16.
// Two uses:
//
//  * FACTOR (segment start state M_s = I + P_s = L L^T): the upper triangle,
//    which starts at zero, carries B = L^{-T} along (row i of the identity
//    solved against the factor, B_ii = 1 / L_ii), so one sweep yields it;
//    the panels of B are stored as three bf16 pieces.  Since
//    M_s^{-1} = B B^T, the whitened rows Y = sqrt(c) X_s B give the segment's
//    problem c X_s M_s^{-1} X_s^T = Y Y^T.
//  * INSEG (one segment): G' = Y Y^T (Y in three pieces, six piece
//    products) is accumulated straight into TMEM, I + G' is factored in
//    place, and the excess of each column gives dR_t = log1p(e_t) / 2.
#pragma once

#include "tc.cuh"

namespace dbc {
namespace cr {

struct TmemChol {
    static constexpr int NT = 256;
    static constexpr uint32_t PIECE = 256 * 128;          // 256-row x 64-K bf16 tile
    static constexpr uint32_t PANEL = 3 * PIECE;          // staged panel (three pieces)
    static constexpr uint32_t GSTAGE = 3 * PIECE;         // G' GEMM stage: the three pieces of Y, 64 K
    static constexpr uint32_t REGION = (2 * GSTAGE > PANEL) ? 2 * GSTAGE : PANEL;
    static constexpr size_t SMEM = REGION + 1024;
};

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

// Stages 16 values of one row as three K-major pieces (K = 16: the first two
// 16-byte chunks of the row's 128-byte line in each 256-row tile).
__device__ __forceinline__ void stage_row16(uint32_t region, int row, const float (&a)[16]) {
#pragma unroll
    for (int k8 = 0; k8 < 2; ++k8) {
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
    }
}

// D[block rows, columns j1 ..) -= sum of the six piece products over K = 16:
// A = staged rows a_row0 .. +128, B = staged rows b_row0 .. +N.
__device__ __forceinline__ void issue_split_mma_k16(uint32_t d_tmem, uint32_t region, int a_row0, int b_row0,
                                                    uint32_t idesc) {
#pragma unroll
    for (int pr = 0; pr < 6; ++pr) {
        const uint32_t pa = region + (uint32_t)pair_a(pr) * TmemChol::PIECE + (uint32_t)a_row0 * 128;
        const uint32_t pb = region + (uint32_t)pair_b(pr) * TmemChol::PIECE + (uint32_t)b_row0 * 128;
        tc::mma_bf16(d_tmem, tc::sdesc(pa, 16, 1024), tc::sdesc(pb, 16, 1024), idesc, 1u);
    }
}

// Runtime N of the negated trailing update (N = 256 - j1, a multiple of 64).
__device__ __forceinline__ uint32_t idesc_neg(int N) { return tc::idesc_bf16(128, N, false, false, true); }

template <bool FACTOR>
__global__ void __launch_bounds__(TmemChol::NT, 1) tmem_chol_kernel(
    Segs S, const float *__restrict__ Pbuf, __nv_bfloat16 *Bscr, const __nv_bfloat16 *__restrict__ Y3,
    int64_t N, float *dR, int32_t *st) {
    constexpr int D = 256;
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[2];
    __shared__ uint32_t tmem_base;
    __shared__ __align__(16) float s_LdT[16][16];   // factored 16 x 16 diagonal block, column-major
    __shared__ __align__(16) float s_rl[16];        // 1 / L_kk of the diagonal block
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int blk = warp >> 2, lb = (warp & 3) * 32;
    const int row = blk * 128 + lb + lane;
    const uint32_t region = (tc::smem_u32(smraw) + 1023u) & ~1023u;
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
            // G' = Y Y^T: per 64-feature chunk the three pieces of the segment's Y rows, six piece
            // products; rows 0..127 only need columns 0..127 (the lower triangle); two stages
            constexpr int NCH = D / 64;
            auto load = [&](int c, uint32_t sb) {
                for (int e = tid; e < 3 * 256 * 8; e += TmemChol::NT) {
                    const int p = e >> 11, r = (e >> 3) & 255, ch = e & 7;
                    const bool in = r < len;
                    const __nv_bfloat16 *gy = Y3 + (size_t)p * N * D + (size_t)(start + (in ? r : 0)) * D + c * 64 + ch * 8;
                    tc::cp_async16(sb + (uint32_t)p * TmemChol::PIECE + tc::kmajor_off(r, ch * 8), gy, in ? 16u : 0u);
                }
            };
            constexpr uint32_t idg0 = tc::idesc_bf16(128, 128, false, false);
            constexpr uint32_t idg1 = tc::idesc_bf16(128, 256, false, false);
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
                    for (int pr = 0; pr < 6; ++pr) {
                        const uint32_t pa = sb + (uint32_t)pair_a(pr) * TmemChol::PIECE;
                        const uint32_t pb = sb + (uint32_t)pair_b(pr) * TmemChol::PIECE;
#pragma unroll
                        for (int b = 0; b < 2; ++b)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                tc::mma_bf16(tbase + (uint32_t)(b * 256),
                                             tc::sdesc(pa + (uint32_t)b * 128 * 128 + kk * 32, 16, 1024),
                                             tc::sdesc(pb + kk * 32, 16, 1024), b == 0 ? idg0 : idg1,
                                             (c > 0 || pr > 0 || kk > 0) ? 1u : 0u);
                    }
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

        // ---------------- 16-column panels
        // Each panel: its 16 TMEM columns -> registers; the 16 x 16 diagonal block is factored by
        // its half-warp with shuffles; every other live row solves its 16 values against it; the
        // values are staged as three bf16 pieces and all later columns are updated by tcgen05 MMAs
        // (negated A, six piece products, K = 16).  Two barriers and one MMA wait per panel.
        __nv_bfloat16 *Bs = FACTOR ? Bscr + (size_t)s * 3 * D * D : nullptr;
        for (int j0 = 0; j0 < n; j0 += 16) {
            const int nb = min(16, n - j0);
            const int j1 = j0 + nb;
            const int ii = row - j0;
            const bool diag = ii >= 0 && ii < 16;
            float v[16];
            __syncwarp();
            tc::tmem_ld16(trow + (uint32_t)j0, v);
            if (FACTOR && diag) {
                // right of its diagonal a row carries B, which only receives contributions from
                // columns at or after its own: what earlier updates left there is dropped
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    if (c > ii) v[c] = 0.f;
            }
            float a[16];
            if (diag) {
                // branch-free (selects only): the half-warp stays converged for its shuffles, and
                // the per-pivot work on the serial path is one broadcast, one rsqrt and one fma;
                // each lane keeps its own pivot's values and writes them afterwards
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
                if (!FACTOR && ii < nb) dR[start + j0 + ii] = 0.5f * log1pf(e_mine);
#pragma unroll
                for (int c = 0; c < 16; ++c) s_LdT[c][ii] = c <= ii ? v[c] : 0.f;
            }
            __syncthreads();
            // rows at or above the block are finished in the in-segment mode
            const bool live = FACTOR || ii >= 16;
            if (live) {
                // right-looking solve against the diagonal block: a[m] is final once the columns
                // before m are applied; a diagonal-block row takes the B role (B_im = 0 for m < ii,
                // B_ii = 1/L_ii); rows above the block carry B, rows below L
                float rl[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 r4 = reinterpret_cast<const float4 *>(s_rl)[j];
                    rl[4 * j] = r4.x; rl[4 * j + 1] = r4.y; rl[4 * j + 2] = r4.z; rl[4 * j + 3] = r4.w;
                }
                const float binv = diag ? 1.f / s_LdT[ii][ii] : 0.f;      // B_ii = 1 / L_ii (IEEE)
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    float am = v[m] * rl[m];
                    if (diag && m <= ii) am = m == ii ? binv : 0.f;
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
            } else {
#pragma unroll
                for (int m = 0; m < 16; ++m) a[m] = 0.f;
            }
            if (FACTOR && row < j1) {
                // B panel -> global pieces (rows >= j1 are zero here and never stored: the loads
                // of the whitening GEMM zero-fill them)
                __nv_bfloat16 *g = Bs + (size_t)row * D + j0;
#pragma unroll
                for (int k8 = 0; k8 < 2; ++k8) {
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
                    *reinterpret_cast<uint4 *>(g + k8 * 8) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
                    *reinterpret_cast<uint4 *>(g + (size_t)D * D + k8 * 8) = make_uint4(mm[0], mm[1], mm[2], mm[3]);
                    *reinterpret_cast<uint4 *>(g + (size_t)2 * D * D + k8 * 8) = make_uint4(ll[0], ll[1], ll[2], ll[3]);
                }
            }
            if (j1 < n) {
                // operand rows of the trailing update: L (rows >= j1), B (factor mode, rows < j1),
                // zero (in-segment mode, rows < j1)
                stage_row16(region, row, a);
                // factor mode: the diagonal rows' B entries right of the panel start from zero.
                // tcgen05.ld/st are warp-collective (.sync.aligned) and a warp may only address its
                // lane group, so the two warps of the block rows' lane group (one per row block)
                // read the columns past the panel and write them back, zeros for the block rows;
                // each takes every other 32 columns, two loads in flight per wait.
                const int gd = (j0 & 127) >> 5, bd = j0 >> 7;     // lane group, row block of the block
                if (FACTOR && (warp & 3) == gd) {                 // warp-uniform
                    __syncwarp();
                    const int lrow = bd * 128 + gd * 32 + lane;   // row of this lane in those columns
                    const bool zero = lrow >= j0 && lrow < j0 + 16;
                    const uint32_t tb = tbase + ((uint32_t)(gd * 32) << 16) + (uint32_t)(bd * 256);
#pragma unroll 1
                    for (int c0 = j1 + 32 * (warp >> 2); c0 < D; c0 += 64) {
                        const bool two = c0 + 16 < D;             // warp-uniform
                        uint32_t r0[16], r1[16] = {};
                        tc::tmem_ld16_nw(tb + (uint32_t)c0, r0);
                        if (two) tc::tmem_ld16_nw(tb + (uint32_t)(c0 + 16), r1);
                        tc::tmem_wait_ld();
                        float t0[16], t1[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            t0[i] = zero ? 0.f : __uint_as_float(r0[i]);
                            t1[i] = zero ? 0.f : __uint_as_float(r1[i]);
                        }
                        tc::tmem_st16(tb + (uint32_t)c0, t0);
                        if (two) tc::tmem_st16(tb + (uint32_t)(c0 + 16), t1);
                    }
                    tc::tmem_wait_st();
                }
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            __syncthreads();
            if (j1 < n) {
                if (tid == 0) {
                    tc::fence_after_sync();
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        if (!FACTOR && (b + 1) * 128 <= j1) continue;
                        // in-segment mode: the first row block only needs its lower triangle (columns < 128)
                        const int nc = (!FACTOR && b == 0) ? 128 - j1 : 256 - j1;
                        issue_split_mma_k16(tbase + (uint32_t)(b * 256 + j1), region, b * 128, j1, idesc_neg(nc));
                    }
                    tc::mma_commit(&mbar[0]);
                }
                ok &= tc::mbar_wait(&mbar[0], ph0, st);
                ph0 ^= 1;
                tc::fence_after_sync();
                ok = __syncthreads_and(ok) != 0;
                if (!ok) break;
            }
        }
        if (!ok) break;

    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

}  // namespace cr
}  // namespace dbc
