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
//    each solved panel is written back to TMEM and B leaves for global memory
//    once, as three bf16 pieces, after the last panel.  Since
//    M_s^{-1} = B B^T, the whitened rows Y = sqrt(c) X_s B give the segment's
//    problem c X_s M_s^{-1} X_s^T = Y Y^T.
//  * INSEG (one segment): G' = Y Y^T (Y in three pieces, six piece
//    products, or three products of the first two pieces for a 64-feature
//    chunk of Y whose rows are all small) is accumulated straight into TMEM,
//    I + G' is factored in place, and the excess of each column gives
//    dR_t = log1p(e_t) / 2.
#pragma once

#include <cuda.h>

#include "tc.cuh"

namespace dbc {
namespace cr {

// 1 / sqrt(x) from the hardware approximation with subnormals flushed: the pivots are 1 + e with
// e >= 0 in exact arithmetic, so the argument is never subnormal and the flush costs nothing.
__device__ __forceinline__ float rsqrt_ftz(float x) {
    float y;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct TmemChol {
    static constexpr int NT = 256;
    static constexpr uint32_t PIECE = 256 * 128;          // 256-row x 64-K bf16 tile
    static constexpr uint32_t PANEL = 3 * PIECE;          // staged panel (three pieces)
    // in-segment Gram: the pieces of Y_c (3 x PIECE), then two operand stages of X (256 x 64 K,
    // K-major) and the three pieces of a 64 x 64 block of B (MN-major)
    static constexpr uint32_t YX_BYTES = 2 * 128 * 128;
    static constexpr uint32_t YSTAGE = YX_BYTES + 3 * 8192;
    static constexpr uint32_t YSTAGE0 = 3 * PIECE;
    static constexpr uint32_t YREGION = YSTAGE0 + 2 * YSTAGE;
    static constexpr uint32_t REGION = (YREGION > 2 * PANEL) ? YREGION : 2 * PANEL;
    static constexpr size_t SMEM = REGION + 1024;
    // A 64-feature chunk Y_c of G' = sum_c Y_c Y_c^T takes three of the six piece products
    // (hi.hi, hi.mid, mid.hi: the two-piece split hi + mid, dropped terms below 2^-16 |y_t||y_u|)
    // when every live row has |y_{t,c}|^2 <= this bound: each dropped entry is then below
    // 2^-16 * 4 = 6e-5, far under the unit floor of I + G', so the leading factor's pivots move by
    // a few parts in 1e5 (measured in float64 emulation on every workload family: dR within 2e-5
    // relative).  Chunks above it (whitened rows the prefix has not yet explained: the first
    // segments of a row) keep all six products.
    static constexpr float Y2_TWO_PIECE = 4.f;
};

// Six piece products of a three-way split (dropped terms are below 2^-24):
// hi.hi, hi.mid, mid.hi, hi.lo, lo.hi, mid.mid.
__device__ __forceinline__ constexpr int pair_a(int i) { return i == 2 ? 1 : (i == 4 ? 2 : (i == 5 ? 1 : 0)); }
__device__ __forceinline__ constexpr int pair_b(int i) { return i == 1 ? 1 : (i == 3 ? 2 : (i == 5 ? 1 : 0)); }

// Two values split at once into three packed bf16x2 pieces (hi, mid, lo): the
// round-to-nearest-even pieces whose sum carries the fp32 value, one paired
// conversion each.
__device__ __forceinline__ void split3x2(float a, float b, uint32_t &h, uint32_t &m, uint32_t &l) {
    const __nv_bfloat162 bh = __floats2bfloat162_rn(a, b);
    const float2 fh = __bfloat1622float2(bh);
    const float ra = a - fh.x, rb = b - fh.y;
    const __nv_bfloat162 bm = __floats2bfloat162_rn(ra, rb);
    const float2 fm = __bfloat1622float2(bm);
    const __nv_bfloat162 bl = __floats2bfloat162_rn(ra - fm.x, rb - fm.y);
    h = *reinterpret_cast<const uint32_t *>(&bh);
    m = *reinterpret_cast<const uint32_t *>(&bm);
    l = *reinterpret_cast<const uint32_t *>(&bl);
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
        for (int q = 0; q < 4; ++q) split3x2(a[k8 * 8 + 2 * q], a[k8 * 8 + 2 * q + 1], hh[q], mm[q], ll[q]);
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

// D[block rows, columns j1 ..) -= sum of the six piece products over K = 16:
// A = staged rows a_row0 .. +128, B = staged rows b_row0 .. +N.
// `dreg` is the descriptor of the staging region's first byte (K-major, SBO 1024).
__device__ __forceinline__ void issue_split_mma_k16(uint32_t d_tmem, uint64_t dreg, int a_row0, int b_row0,
                                                    uint32_t idesc) {
    const uint64_t da = tc::sdesc_add(dreg, (uint32_t)a_row0 * 128), db = tc::sdesc_add(dreg, (uint32_t)b_row0 * 128);
#pragma unroll
    for (int pr = 0; pr < 6; ++pr)
        tc::mma_bf16(d_tmem, tc::sdesc_add(da, (uint32_t)pair_a(pr) * TmemChol::PIECE),
                     tc::sdesc_add(db, (uint32_t)pair_b(pr) * TmemChol::PIECE), idesc, 1u);
}

// Runtime N of the negated trailing update (N = 256 - j1, a multiple of 64).
__device__ __forceinline__ uint32_t idesc_neg(int N) { return tc::idesc_bf16(128, N, false, false, true); }

// Block-wide barrier and AND-vote of the 256 threads (named barrier 1).
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ bool cbar_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.and.pred p, 1, 256, q;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool cbar_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, 1, 256, q;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Pair pi of the in-segment Y GEMM -> (output chunk c, K chunk k), k <= c < 4.
__device__ __forceinline__ void ypair(int pi, int &c, int &k) {
    c = 0;
    k = pi;
    while (k > c) { k -= c + 1; ++c; }
}

// tmP: P as fp32 [segments * 256][256] in 32 x 32 boxes (128-byte swizzle); tmB: B's pieces as bf16
// [segments * 3 * 256][256] in 64 x 64 boxes (128-byte swizzle); tmX: H as bf16 [N][256] in boxes of
// xbox_rows = min(N, 256) positions x 64 features (128-byte swizzle).  All cover this GPU's own memory (no multicast):
// the factor mode loads P and stores B through them, the in-segment mode loads X and B.
template <bool FACTOR>
__global__ void __launch_bounds__(TmemChol::NT, 1) tmem_chol_kernel(
    const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmB,
    const __grid_constant__ CUtensorMap tmX, int xbox_rows, Segs S,
    const float *__restrict__ Pbuf, __nv_bfloat16 *Bscr, const __nv_bfloat16 *__restrict__ Hx, int64_t N,
    float c_rate, float *dR, int32_t *st) {
    constexpr int D = 256;
    extern __shared__ uint8_t smraw[];
    // [0], [1] panel MMA groups; [2] the final drain; [3], [4] Y operand stages consumed; [5] Y chunk done;
    // [6], [7] Y operand stages loaded (TMA bytes)
    __shared__ uint64_t mbar[9];                    // [8]: the factor mode's P boxes landed
    __shared__ uint32_t tmem_base;
    __shared__ __align__(16) float s_LdT[16][16];   // factored 16 x 16 diagonal block, column-major
    __shared__ __align__(16) float s_rl[16];        // 1 / L_kk of the diagonal block
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // MMAs are issued by one thread, lane 0 of warp 7: in-order MMA semantics need a single issuer,
    // and warp 7 is the diagonal-block warp of only the last two panels, so the issue time is spent
    // while the other warps factor the next diagonal block
    const bool issuer = tid == 7 * 32;
    const int blk = warp >> 2, lb = (warp & 3) * 32;
    const int row = blk * 128 + lb + lane;
    const uint32_t region = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    const uint64_t dregion = tc::sdesc(region, 16, 1024);      // K-major tiles of the region
    if (warp == 0) tc::tmem_alloc(&tmem_base, 512);
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) tc::mbar_init(&mbar[i], 1);
        tc::mbar_init(&mbar[8], 1);
        tc::tma_prefetch_desc(FACTOR ? &tmP : &tmX);
        tc::tma_prefetch_desc(&tmB);
        for (int i = 6; i < 8; ++i) tc::mbar_init(&mbar[i], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const int nseg = *S.nseg;
    constexpr int NPAIR = 10;
    constexpr uint32_t idy = tc::idesc_bf16(128, 64, false, true);
    constexpr uint32_t idg0 = tc::idesc_bf16(128, 128, false, false);
    constexpr uint32_t idg1 = tc::idesc_bf16(128, 256, false, false);

    {
        // ================= thread (warp w, lane l) owns row (w/4)*128 + (w%4)*32 + l
        const uint32_t trow = tbase + ((uint32_t)lb << 16) + (uint32_t)(blk * 256);
        uint32_t ph0 = 0, ph1 = 0;      // mbarrier phases (uniform across the compute threads)
        uint32_t phs = 0, phy = 0, pf = 0;   // phs, pf: bit q = parity of the next wait on stage q
        uint32_t pph = 0;                    // parity of the next wait on the P boxes
        bool ok = true;
        // A timeout makes `ok` false: every later wait and MMA is skipped (commits still arrive),
        // and the block-wide votes keep all threads on the same path to the end.
        for (int s = blockIdx.x; s < nseg; s += gridDim.x) {
            const int len = S.len[s];
            const int64_t start = S.start[s];
            const int n = FACTOR ? D : len;

            // ---------------- load the matrix into TMEM
            if (FACTOR) {
                // The c-scaled prefix Gram's lower triangle at 32-column granularity comes in with TMA:
                // box (q, rb) = rows rb*32 .. +31 x columns q*32 .. +31 for rb >= q, 36 boxes of 4 KB,
                // all in flight at once, in slots ordered by q then rb.  Each thread then moves its own
                // row into TMEM (zeros right of its diagonal, where B = L^{-T} accumulates).
                auto slot = [](int q, int rb) { return 8 * q - (q * (q - 1)) / 2 + (rb - q); };
                if (tid == 0 && ok) {
                    tc::mbar_arrive_expect_tx(&mbar[8], 36u * 4096u);
                    for (int q = 0; q < 8; ++q)
                        for (int rb = q; rb < 8; ++rb)
                            tc::tma_load_2d(region + (uint32_t)slot(q, rb) * 4096u, &tmP, &mbar[8], q * 32,
                                            s * D + rb * 32);
                }
                if (ok) ok = tc::mbar_wait(&mbar[8], pph, st);
                pph ^= 1u;
                const uint8_t *pbox = smraw + (region - tc::smem_u32(smraw));
                const int rb = row >> 5, rin = row & 31;
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    const bool any = ok && q <= rb;                    // warp-uniform
                    float x[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (any)
                            f = *reinterpret_cast<const float4 *>(pbox + (size_t)slot(q, rb) * 4096 + rin * 128 +
                                                                  ((c ^ (rin & 7)) * 16));
                        x[4 * c] = f.x; x[4 * c + 1] = f.y; x[4 * c + 2] = f.z; x[4 * c + 3] = f.w;
                    }
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        float v[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = (q * 32 + j * 16 + i <= row) ? x[j * 16 + i] : 0.f;
                        tc::tmem_st16(trow + (uint32_t)(q * 32 + j * 16), v);
                    }
                }
                tc::tmem_wait_st();
            } else {
                // G' = Y Y^T with the whitened rows Y = sqrt(c) X_s B_s formed here, 64 features at
                // a time: Y_c = X_s B_s[:, chunk c] accumulates in the TMEM columns 128..255 (free in
                // this mode: the first row block only uses its lower triangle), over the K chunks
                // k <= c (B is upper triangular) with X and the three pieces of B streamed through
                // two cp.async stages; Y_c is then split into three bf16 pieces in shared memory and
                // G' += Y_c Y_c^T (six piece products) is issued while the next chunk's operands load.
                // The issuing thread loads the operand stages with TMA: X_s's 256 positions x 64
                // features of K chunk k (one box; positions past the segment, whose Y rows never reach
                // the leading n x n block that is factored, arrive too, or as zeros past the end of H)
                // and the three pieces of B's 64 x 64 block (k, c), every one of which the factor mode
                // stored.
                auto tload = [&](int pi, int q) {
                    int c, k;
                    ypair(pi, c, k);
                    const uint32_t sa = region + TmemChol::YSTAGE0 + (uint32_t)q * TmemChol::YSTAGE;
                    tc::mbar_arrive_expect_tx(&mbar[6 + q], (uint32_t)xbox_rows * 128u + 3u * 8192u);
                    tc::tma_load_2d(sa, &tmX, &mbar[6 + q], k * 64, (int)start);
                    for (int p = 0; p < 3; ++p)
                        tc::tma_load_2d(sa + TmemChol::YX_BYTES + (uint32_t)p * 8192u, &tmB, &mbar[6 + q], c * 64,
                                        (s * 3 + p) * D + k * 64);
                };
                const float sc = sqrtf(c_rate);
                if (issuer && ok) tload(0, 0);
                for (int pi = 0; pi < NPAIR; ++pi) {
                    int c, k;
                    ypair(pi, c, k);
                    if (pi + 1 < NPAIR) {
                        const int q = (pi + 1) & 1;
                        if (pi + 1 >= 2) {                                   // stage q was read by pair pi - 1
                            if (issuer && ok) ok = tc::mbar_wait(&mbar[3 + q], (phs >> q) & 1u, st);
                            phs ^= 1u << q;
                        }
                        if (issuer && ok) tload(pi + 1, q);
                    }
                    if (issuer) {
                        if (ok) ok = tc::mbar_wait(&mbar[6 + (pi & 1)], (pf >> (pi & 1)) & 1u, st);
                        pf ^= 1u << (pi & 1);
                        if (ok) {
                            tc::fence_after_sync();
                            const uint32_t sa = region + TmemChol::YSTAGE0 + (uint32_t)(pi & 1) * TmemChol::YSTAGE;
                            const uint64_t dxa = tc::sdesc(sa, 16, 1024);                        // X, K-major
                            const uint64_t dbb = tc::sdesc(sa + TmemChol::YX_BYTES, 8192, 1024);  // B, MN-major
#pragma unroll
                            for (int b = 0; b < 2; ++b)
#pragma unroll
                                for (int p = 0; p < 3; ++p)
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        tc::mma_bf16(tbase + (uint32_t)(128 + b * 64),
                                                     tc::sdesc_add(dxa, (uint32_t)b * 128 * 128 + kk * 32),
                                                     tc::sdesc_add(dbb, (uint32_t)p * 8192 + kk * 2048), idy,
                                                     (k > 0 || p > 0 || kk > 0) ? 1u : 0u);
                        }
                        tc::mma_commit(&mbar[3 + (pi & 1)]);
                        if (k == c) tc::mma_commit(&mbar[5]);
                    }
                    if (k == c) {
                        // Y_c complete (and with it every earlier MMA, so the pieces buffer is free)
                        if (ok) ok = tc::mbar_wait(&mbar[5], phy, st);
                        phy ^= 1;
                        tc::fence_after_sync();
                        ok = __all_sync(0xffffffffu, ok);
                        bool big = false;                  // this row's |Y_c|^2 above the two-piece bound
                        if (ok) {
                            float a64[64];
                            float s2 = 0.f;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                float v16[16];
                                tc::tmem_ld16(tbase + ((uint32_t)lb << 16) + (uint32_t)(128 + blk * 64 + q * 16), v16);
#pragma unroll
                                for (int i = 0; i < 16; ++i) {
                                    a64[q * 16 + i] = sc * v16[i];
                                    s2 = fmaf(a64[q * 16 + i], a64[q * 16 + i], s2);
                                }
                            }
                            big = row < n && !(s2 <= TmemChol::Y2_TWO_PIECE);
                            stage_row(region, row, a64, nullptr, 0);
                        }
                        tc::fence_async_smem();
                        tc::fence_before_sync();
                        ok = cbar_and(ok);
                        const int npr = cbar_or(big) ? 6 : 3;
                        if (issuer && ok) {
                            tc::fence_after_sync();
                            const uint64_t dyp = tc::sdesc(region, 16, 1024);
#pragma unroll
                            for (int pr = 0; pr < 6; ++pr) {
                                if (pr >= npr) break;
                                const uint32_t pa = (uint32_t)pair_a(pr) * TmemChol::PIECE;
                                const uint32_t pb = (uint32_t)pair_b(pr) * TmemChol::PIECE;
#pragma unroll
                                for (int b = 0; b < 2; ++b)
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        tc::mma_bf16(tbase + (uint32_t)(b * 256),
                                                     tc::sdesc_add(dyp, pa + (uint32_t)b * 128 * 128 + kk * 32),
                                                     tc::sdesc_add(dyp, pb + kk * 32), b == 0 ? idg0 : idg1,
                                                     (c > 0 || pr > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                    }
                }
                // G' complete; the last two stage commits are consumed so every commit has its wait
                if (issuer) tc::mma_commit(&mbar[5]);
                if (ok) ok = tc::mbar_wait(&mbar[5], phy, st);
                phy ^= 1;
                for (int q = 0; q < 2; ++q) {
                    if (ok) ok = tc::mbar_wait(&mbar[3 + q], (phs >> q) & 1u, st);
                    phs ^= 1u << q;
                }
            }
            tc::fence_before_sync();
            ok = cbar_and(ok);
            tc::fence_after_sync();

            // ---------------- 16-column panels with a one-panel look-ahead
            // Panel j: its 16 TMEM columns -> registers; the 16 x 16 diagonal block is factored by its
            // half-warp with shuffles; every other live row solves its 16 values against it; the
            // values are staged as three bf16 pieces (two staging buffers, alternating) and the issuing
            // thread issues the negated K = 16 tcgen05 MMAs of the trailing update in two groups: the next panel's 16 columns (committed to mbar[0]) and then every later column
            // (committed to mbar[1]).  Panel j+1 waits for mbar[0] only, so the bulk of the update
            // runs under its factorization.  In the factor mode the rows of the diagonal block must
            // start their B entries right of the panel from zero: the other warp of their TMEM lane
            // group resets those entries once the previous panel's bulk update has landed, after its
            // own solve.
            const int npan = (n + 15) / 16;
            // phase bookkeeping: panel j < npan - 1 commits once to each barrier; completion k of a
            // barrier is awaited with parity (base + k) & 1
            const uint32_t base0 = ph0, base1 = ph1;
            for (int j = 0; j < npan; ++j) {
                const int j0 = 16 * j;
                const int nb = min(16, n - j0);
                const int j1 = j0 + nb;
                const int ii = row - j0;
                const bool diag = ii >= 0 && ii < 16;
                const uint32_t R = region + (uint32_t)(j & 1) * TmemChol::PANEL;
                if (j > 0) {
                    // the previous panel's update of these 16 columns (and every earlier MMA) has
                    // landed; a timeout is acted on at the next vote
                    if (ok) ok = tc::mbar_wait(&mbar[0], (base0 + (uint32_t)(j - 1)) & 1u, st);
                    tc::fence_after_sync();
                }
                float v[16];
                __syncwarp();
                tc::tmem_ld16(trow + (uint32_t)j0, v);
                const int gd = (j0 & 127) >> 5, bd = j0 >> 7;     // lane group, row block of the block rows
                if (FACTOR && diag) {
                    // right of its diagonal a row carries B, which only receives contributions from
                    // columns at or after its own: what earlier updates left there is dropped
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (c > ii) v[c] = 0.f;
                }
                float a[16];
                if (diag) {
                    // Four pivots per step (branch-free, selects only, so the half-warp stays converged
                    // for its shuffles): every lane takes the 4 x 4 diagonal block of columns c .. c+3
                    // (ten broadcasts at once) and factors it itself, solves its own row's four values
                    // against it (l = L4^-1 x) and applies the four columns to the rest of its row as
                    // v -= g . w with g = L4^-T l and w the four values of the other row, so the serial
                    // path per four pivots is one round of shuffles, four rsqrt and a few fma.  Every
                    // lane updates all 16 entries of its row: those right of its own diagonal become
                    // scratch (no other lane reads them; the factor mode restores its zeros below).
                    // Each lane keeps its own pivot's values and writes them afterwards.
                    const int lb0 = lane & 16;
                    const unsigned mask = 0xFFFFu << lb0;
                    float rl_mine = 1.f, e_mine = 0.f;
#pragma unroll
                    for (int c = 0; c < 16; c += 4) {
                        float a[4][4];                                       // a[p][q], q <= p
#pragma unroll
                        for (int p = 0; p < 4; ++p)
#pragma unroll
                            for (int q = 0; q <= p; ++q) a[p][q] = __shfl_sync(mask, v[c + q], lb0 + c + p);
                        // L4 (unit-free: the diagonal of I + a is 1 + e)
                        const float r0 = rsqrt_ftz(1.f + a[0][0]);
                        const float L10 = a[1][0] * r0, L20 = a[2][0] * r0, L30 = a[3][0] * r0;
                        const float e1 = fmaf(-L10, L10, a[1][1]);
                        const float r1 = rsqrt_ftz(1.f + e1);
                        const float L21 = fmaf(-L20, L10, a[2][1]) * r1, L31 = fmaf(-L30, L10, a[3][1]) * r1;
                        const float e2 = fmaf(-L21, L21, fmaf(-L20, L20, a[2][2]));
                        const float r2 = rsqrt_ftz(1.f + e2);
                        const float L32 = fmaf(-L31, L21, fmaf(-L30, L20, a[3][2])) * r2;
                        const float e3 = fmaf(-L32, L32, fmaf(-L31, L31, fmaf(-L30, L30, a[3][3])));
                        const float r3 = rsqrt_ftz(1.f + e3);
                        // this row's factor entries in the four columns
                        const float l0 = v[c] * r0;
                        const float l1 = fmaf(-l0, L10, v[c + 1]) * r1;
                        const float l2 = fmaf(-l1, L21, fmaf(-l0, L20, v[c + 2])) * r2;
                        const float l3 = fmaf(-l2, L32, fmaf(-l1, L31, fmaf(-l0, L30, v[c + 3]))) * r3;
                        const float g3 = l3 * r3;
                        const float g2 = fmaf(-g3, L32, l2) * r2;
                        const float g1 = fmaf(-g3, L31, fmaf(-g2, L21, l1)) * r1;
                        const float g0 = fmaf(-g3, L30, fmaf(-g2, L20, fmaf(-g1, L10, l0))) * r0;
#pragma unroll
                        for (int c2 = c + 4; c2 < 16; ++c2) {
                            const float w0 = __shfl_sync(mask, v[c], lb0 + c2);
                            const float w1 = __shfl_sync(mask, v[c + 1], lb0 + c2);
                            const float w2 = __shfl_sync(mask, v[c + 2], lb0 + c2);
                            const float w3 = __shfl_sync(mask, v[c + 3], lb0 + c2);
                            v[c2] = fmaf(-g3, w3, fmaf(-g2, w2, fmaf(-g1, w1, fmaf(-g0, w0, v[c2]))));
                        }
                        const float e0 = a[0][0];
                        v[c] = ii == c ? (1.f + e0) * r0 : l0;                  // L_cc on its row
                        v[c + 1] = ii == c + 1 ? (1.f + e1) * r1 : l1;
                        v[c + 2] = ii == c + 2 ? (1.f + e2) * r2 : l2;
                        v[c + 3] = ii == c + 3 ? (1.f + e3) * r3 : l3;
                        rl_mine = ii == c ? r0 : (ii == c + 1 ? r1 : (ii == c + 2 ? r2 : (ii == c + 3 ? r3 : rl_mine)));
                        e_mine = ii == c ? e0 : (ii == c + 1 ? e1 : (ii == c + 2 ? e2 : (ii == c + 3 ? e3 : e_mine)));
                    }
                    if (FACTOR) {
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            if (c > ii) v[c] = 0.f;
                    }
                    s_rl[ii] = rl_mine;
                    if (!FACTOR && ii < nb && ok && dcheck(start + j0 + ii < N, st))
                        dR[start + j0 + ii] = 0.5f * log1pf(e_mine);
#pragma unroll
                    for (int c = 0; c < 16; ++c) s_LdT[c][ii] = c <= ii ? v[c] : 0.f;
                }
                ok = cbar_and(ok);
                // rows at or above the block are finished in the in-segment mode
                const bool live = FACTOR || ii >= 16;
                if (live) {
                    // right-looking solve against the diagonal block: a[m] is final once the columns
                    // before m are applied; a diagonal-block row takes the B role (B_im = 0 for m < ii,
                    // B_ii = 1/L_ii); rows above the block carry B, rows below L
                    float rl[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 r4 = reinterpret_cast<const float4 *>(s_rl)[q];
                        rl[4 * q] = r4.x; rl[4 * q + 1] = r4.y; rl[4 * q + 2] = r4.z; rl[4 * q + 3] = r4.w;
                    }
                    const float binv = diag ? 1.f / s_LdT[ii][ii] : 0.f;      // B_ii = 1 / L_ii (IEEE)
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        float am = v[m] * rl[m];
                        if (diag && m <= ii) am = m == ii ? binv : 0.f;
                        a[m] = am;
                        const float4 *lr = reinterpret_cast<const float4 *>(&s_LdT[m][0]);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (4 * q + 3 > m) {
                                const float4 l = lr[q];
                                if (4 * q + 0 > m) v[4 * q + 0] = fmaf(-am, l.x, v[4 * q + 0]);
                                if (4 * q + 1 > m) v[4 * q + 1] = fmaf(-am, l.y, v[4 * q + 1]);
                                if (4 * q + 2 > m) v[4 * q + 2] = fmaf(-am, l.z, v[4 * q + 2]);
                                v[4 * q + 3] = fmaf(-am, l.w, v[4 * q + 3]);
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 16; ++m) a[m] = 0.f;
                }
                if (FACTOR && j1 < n && warp == (1 - bd) * 4 + gd) {
                    // the reset helper, the other warp of the block rows' TMEM lane quarter: right of the
                    // panel the block rows carry B, which restarts from zero once the previous panel's
                    // bulk update has landed (done here, after the solve, so that its wait is hidden;
                    // this panel's updates of those entries are issued after the next vote).  Stores of
                    // zeros to those 16 lanes only, nothing read back.
                    bool okh = ok;
                    if (j > 0 && okh) {
                        okh = tc::mbar_wait(&mbar[1], (base1 + (uint32_t)(j - 1)) & 1u, st);   // previous bulk update
                        tc::fence_after_sync();
                    }
                    okh = __all_sync(0xffffffffu, okh);
                    if (okh) {
                        const uint32_t tz = tbase + ((uint32_t)(gd * 32 + (j0 & 31)) << 16) + (uint32_t)(bd * 256);
                        int c0 = j1;
#pragma unroll 1
                        for (; c0 + 32 <= D; c0 += 32) tc::tmem_st_zero16x32(tz + (uint32_t)c0);
                        if (c0 < D) tc::tmem_st_zero16x16(tz + (uint32_t)c0);
                        tc::tmem_wait_st();
                    }
                    ok &= okh;
                }
                if (FACTOR) {
                    // the panel's final values stay in TMEM (B right of the diagonal, zero left of it
                    // in the block rows, L below); B leaves for global memory once, after the panels
                    tc::tmem_st16(trow + (uint32_t)j0, a);
                    tc::tmem_wait_st();
                }
                if (j1 < n) {
                    // the row's 16 values as three bf16 pieces: operand rows of the trailing update (L
                    // for rows >= j1, B in the factor mode for rows < j1, zero in the in-segment mode)
                    uint32_t hh[8], mm[8], ll[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) split3x2(a[2 * q], a[2 * q + 1], hh[q], mm[q], ll[q]);
#pragma unroll
                    for (int k8 = 0; k8 < 2; ++k8) {
                        const uint32_t off = tc::kmajor_off(row, k8 * 8);
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(R + off), "r"(hh[4 * k8]),
                                     "r"(hh[4 * k8 + 1]), "r"(hh[4 * k8 + 2]), "r"(hh[4 * k8 + 3])
                                     : "memory");
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(R + TmemChol::PIECE + off),
                                     "r"(mm[4 * k8]), "r"(mm[4 * k8 + 1]), "r"(mm[4 * k8 + 2]), "r"(mm[4 * k8 + 3])
                                     : "memory");
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(R + 2 * TmemChol::PIECE + off),
                                     "r"(ll[4 * k8]), "r"(ll[4 * k8 + 1]), "r"(ll[4 * k8 + 2]), "r"(ll[4 * k8 + 3])
                                     : "memory");
                    }
                }
                if (j1 < n) {
                    tc::fence_async_smem();
                    tc::fence_before_sync();
                    ok = cbar_and(ok);                  // the whole panel is staged
                    if (issuer) {
                        const uint64_t dR_reg = tc::sdesc_add(dregion, (uint32_t)(j & 1) * TmemChol::PANEL);
                        if (ok) {
                            tc::fence_after_sync();
                            // the next panel's 16 columns first, then everything right of them
#pragma unroll
                            for (int b = 0; b < 2; ++b) {
                                if (!FACTOR && (b + 1) * 128 <= j1) continue;
                                issue_split_mma_k16(tbase + (uint32_t)(b * 256 + j1), dR_reg, b * 128, j1,
                                                    idesc_neg(16));
                            }
                        }
                        tc::mma_commit(&mbar[0]);
                        if (ok) {
#pragma unroll
                            for (int b = 0; b < 2; ++b) {
                                if (!FACTOR && (b + 1) * 128 <= j1) continue;
                                // in-segment mode: the first row block only needs its lower triangle
                                const int nc = ((!FACTOR && b == 0) ? 128 : 256) - j1 - 16;
                                if (nc > 0)
                                    issue_split_mma_k16(tbase + (uint32_t)(b * 256 + j1 + 16), dR_reg, b * 128,
                                                        j1 + 16, idesc_neg(nc));
                            }
                        }
                        tc::mma_commit(&mbar[1]);
                    }
                }
            }
            // every MMA of this segment has landed before the next segment (or the exit) reuses TMEM
            if (npan > 1) {
                if (ok) ok = tc::mbar_wait(&mbar[1], (base1 + (uint32_t)(npan - 2)) & 1u, st);
                tc::fence_after_sync();
            }
            ph0 = (base0 + (uint32_t)(npan - 1)) & 1u;
            ph1 = (base1 + (uint32_t)(npan - 1)) & 1u;
            ok = cbar_and(ok);
            if (FACTOR && ok) {
                // B = L^{-T} (TMEM upper triangle with the diagonal) -> three bf16 pieces in global
                // memory, 64 columns at a time: each thread splits its row (zero left of the diagonal)
                // into shared memory in the 128-byte swizzled layout of a 64 x 64 box (alternating
                // between two staging buffers), and one thread stores the boxes with TMA.  Rows below
                // a chunk's last panel are never read by the whitening loads and are not stored.
#pragma unroll 1
                for (int q = 0; q < D / 64; ++q) {
                    const uint32_t stgb = region + (uint32_t)(q & 1) * (3u * 256u * 128u);
                    uint8_t *stg = smraw + (stgb - tc::smem_u32(smraw));
                    // rows at or below the chunk's end hold zeros here and are not stored (warp-uniform:
                    // a warp owns 32 consecutive rows)
                    const bool live_q = row < (q + 1) * 64;
#pragma unroll 1
                    for (int h = 0; h < (live_q ? 4 : 0); ++h) {
                        float v16[16];
                        tc::tmem_ld16(trow + (uint32_t)(q * 64 + h * 16), v16);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (q * 64 + h * 16 + i < row) v16[i] = 0.f;
                        uint32_t hh[8], mm[8], ll[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) split3x2(v16[2 * k], v16[2 * k + 1], hh[k], mm[k], ll[k]);
#pragma unroll
                        for (int c2 = 0; c2 < 2; ++c2) {
                            const int ch = (h * 2 + c2) ^ (row & 7);
                            const size_t o = (size_t)row * 128 + ch * 16;
                            *reinterpret_cast<uint4 *>(stg + o) =
                                make_uint4(hh[4 * c2], hh[4 * c2 + 1], hh[4 * c2 + 2], hh[4 * c2 + 3]);
                            *reinterpret_cast<uint4 *>(stg + 256 * 128 + o) =
                                make_uint4(mm[4 * c2], mm[4 * c2 + 1], mm[4 * c2 + 2], mm[4 * c2 + 3]);
                            *reinterpret_cast<uint4 *>(stg + 2 * 256 * 128 + o) =
                                make_uint4(ll[4 * c2], ll[4 * c2 + 1], ll[4 * c2 + 2], ll[4 * c2 + 3]);
                        }
                    }
                    tc::fence_async_smem();
                    cbar();
                    if (tid == 0) {
                        for (int p = 0; p < 3; ++p)
                            for (int rbk = 0; rbk <= q; ++rbk)
                                asm volatile(
                                    "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];"
                                    ::"l"(&tmB), "r"(q * 64), "r"((s * 3 + p) * D + rbk * 64),
                                    "r"(stgb + (uint32_t)p * 256u * 128u + (uint32_t)rbk * 64u * 128u)
                                    : "memory");
                        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                        // the stores of the previous chunk have read their buffer, which the next chunk
                        // refills
                        asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                    }
                    cbar();
                }
                // the region is reused next: the stores must have read it (their writes may still be in
                // flight; they are complete when the kernel is)
                if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                cbar();
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (issuer) {
        // MMAs still in flight (only after a timeout) finish before the tensor memory is freed
        // (a commit tracks the MMAs of the thread that issued them)
        tc::mma_commit(&mbar[2]);
        tc::mbar_wait(&mbar[2], 0, st);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

}  // namespace cr
}  // namespace dbc
