// Segment Grams and their float64 exclusive prefix in one pass (d = 256, bf16).
//
// The start state of segment s of a row is M_s = I + c P_s with
// P_s = sum over the row's earlier segments s' of X_s'^T X_s' (ByteFlow summary,
// "Prerequisites: lossy coding rate": M_t = I + c sum_{i<=t} h_i h_i^T, cut at
// the segment starts).  One CTA owns one row and one 128 x TN tile of the
// lower triangle of the 256 x 256 matrix and walks the row's segments in
// order:
//   * a producer warp streams the segment's positions in boxes of 64
//     positions x 64 features with TMA (128-byte swizzle, tensor map over this
//     GPU's own memory, no multicast) into a ring of shared-memory stages deep
//     enough for about two segments, so the loads of the next segment are in
//     flight while this one is multiplied;
//   * one thread of the MMA warp issues tcgen05 MMAs G_s[tile] = X_s^T X_s
//     (both operands MN-major: positions are K), bf16 x bf16 products exact,
//     fp32 accumulation in TMEM, two accumulator buffers so that the next
//     segment's MMAs overlap this segment's epilogue;
//   * eight epilogue warps read the tile from TMEM, store c * (running sum)
//     as P_s (fp32, the exclusive prefix) and add G_s to the running sum,
//     which each thread keeps for its row and columns as a compensated fp32
//     pair (hi + lo, about 48 significant bits: every addition's exact error
//     is carried in lo), as accurate here as float64 and far cheaper.
// The running sum may start from a carried float64 state (streams) and is
// then written back (the whole symmetric matrix: off-diagonal tiles also
// write their transpose).  Every mbarrier wait is bounded; a role that gives up
// flags DBC_ERR_TIMEOUT and stops, and the CTA drains its outstanding copies
// and MMAs (bounded) before it frees its tensor memory.
#pragma once

#include <cuda.h>

#include "tc.cuh"

namespace dbc {
namespace cr {

template <int TN>
struct GramPrefixCfg {
    static constexpr int D = 256;
    static constexpr int TILES = TN == 64 ? 6 : 3;        // lower-triangle 128 x TN tiles
    static constexpr int KC = 64;                         // positions per stage
    static constexpr int NS = TN == 64 ? 8 : 6;           // stages: about two segments in flight
    static constexpr uint32_t BOX = 64 * 128;             // 64 positions x 64 features, bf16
    static constexpr uint32_t A_BYTES = 2 * BOX;          // 128 features
    static constexpr uint32_t B_BYTES = (TN / 64) * BOX;  // TN features (off-diagonal tiles only)
    static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
    static constexpr int NT = 320;                        // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
    static constexpr int CPT = TN / 2;                    // columns per epilogue thread
    static constexpr size_t SMEM = NS * STAGE + 1024;
};

// Tile t of the lower triangle: row block b (features b*128 ..) and column block n (features n*TN ..).
template <int TN>
__device__ __forceinline__ void gp_tile(int t, int &b, int &n) {
    if (TN == 64) {
        b = t < 2 ? 0 : 1;
        n = t < 2 ? t : t - 2;
    } else {
        b = t == 0 ? 0 : 1;
        n = t == 2 ? 1 : 0;
    }
}

template <int TN>
__global__ void __launch_bounds__(GramPrefixCfg<TN>::NT, 1) gram_prefix_kernel(
    const __grid_constant__ CUtensorMap tmH, Segs S, int64_t rows, float *P, double *state, double c,
    int32_t *st) {
    using C = GramPrefixCfg<TN>;
    constexpr int D = C::D;
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t full[C::NS], empty[C::NS], acc_full[2], acc_empty[2], drain;
    __shared__ uint32_t tmem_base;
    __shared__ int s_consumed;                 // stages the MMA warp has consumed
    constexpr int kSegCache = 256;             // segments of a row whose table is cached in shared memory
    __shared__ int64_t s_start[kSegCache];
    __shared__ int32_t s_len[kSegCache];
    const int r = blockIdx.x / C::TILES, t = blockIdx.x % C::TILES;
    if (r >= rows) return;
    int b, n;
    gp_tile<TN>(t, b, n);
    const bool diag = n * TN >= b * 128 && n * TN < b * 128 + 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    const int s0 = S.row_seg0[r], s1 = S.row_seg0[r + 1];
    for (int i = tid; i < s1 - s0 && i < kSegCache; i += C::NT) {
        s_start[i] = S.start[s0 + i];
        s_len[i] = S.len[s0 + i];
    }
    if (warp == 1) tc::tmem_alloc(&tmem_base, 2 * TN);
    if (tid == 0) {
        for (int i = 0; i < C::NS; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&acc_full[i], 1);
            tc::mbar_init(&acc_empty[i], 8);
        }
        tc::mbar_init(&drain, 1);
        s_consumed = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmH);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    int issued = 0;                            // producer: stages issued (thread 0 only)

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            bool ok = true;
            for (int s = s0; s < s1 && ok; ++s) {
                const int len = s - s0 < kSegCache ? s_len[s - s0] : S.len[s];
                const int64_t start = s - s0 < kSegCache ? s_start[s - s0] : S.start[s];
                for (int cc = 0; cc * C::KC < len && ok; ++cc) {
                    const int slot = issued % C::NS;
                    if (issued >= C::NS) ok = tc::mbar_wait(&empty[slot], (uint32_t)((issued / C::NS) - 1) & 1u, st);
                    if (!ok) break;
                    const uint32_t sb = base + (uint32_t)slot * C::STAGE;
                    const int y = (int)(start + cc * C::KC);
                    tc::mbar_arrive_expect_tx(&full[slot], diag ? C::A_BYTES : C::STAGE);
                    tc::tma_load_2d(sb, &tmH, &full[slot], b * 128, y);
                    tc::tma_load_2d(sb + C::BOX, &tmH, &full[slot], b * 128 + 64, y);
                    if (!diag)
                        for (int q = 0; q < TN / 64; ++q)
                            tc::tma_load_2d(sb + C::A_BYTES + q * C::BOX, &tmH, &full[slot], n * TN + q * 64, y);
                    ++issued;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issue (lane 0), tail zeroing (whole warp)
        constexpr uint32_t idesc = tc::idesc_bf16(128, TN, true, true);
        bool ok = true;
        int it = 0, seg_i = 0;
        for (int s = s0; s < s1 && ok; ++s, ++seg_i) {
            const int len = s - s0 < kSegCache ? s_len[s - s0] : S.len[s];
            const int buf = seg_i & 1;
            if (seg_i >= 2) ok = tc::mbar_wait(&acc_empty[buf], (uint32_t)((seg_i >> 1) - 1) & 1u, st);
            ok = __all_sync(0xffffffffu, ok);              // warp-uniform decisions only
            if (!ok) break;
            tc::fence_after_sync();
            for (int cc = 0; cc * C::KC < len; ++cc, ++it) {
                const int slot = it % C::NS;
                ok = __all_sync(0xffffffffu, tc::mbar_wait(&full[slot], (uint32_t)(it / C::NS) & 1u, st));
                if (!ok) break;
                const int valid = min(C::KC, len - cc * C::KC);
                const uint32_t sb = base + (uint32_t)slot * C::STAGE;
                const int ksteps = (valid + 15) >> 4;
                if (valid & 15) {
                    // positions past the segment end inside the last K step read as zero rows
                    // (a row of a box is one position's 128 bytes, whatever the swizzle)
                    const int z0 = valid, z1 = ksteps * 16;
                    const int nbox = diag ? 2 : 2 + TN / 64;
                    for (int e = lane; e < (z1 - z0) * nbox * 8; e += 32) {
                        const int row = z0 + e / (nbox * 8), rest = e % (nbox * 8);
                        const int bx = rest >> 3, ch = rest & 7;
                        asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(
                                         sb + (uint32_t)bx * C::BOX + (uint32_t)row * 128 + ch * 16),
                                     "r"(0)
                                     : "memory");
                    }
                    tc::fence_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    tc::fence_after_sync();
                    const uint32_t bb = diag ? sb + (uint32_t)((n * TN - b * 128) / 64) * C::BOX : sb + C::A_BYTES;
                    for (int kk = 0; kk < ksteps; ++kk)
                        tc::mma_bf16(tbase + (uint32_t)(buf * TN), tc::sdesc(sb + kk * 2048, C::BOX, 1024),
                                     tc::sdesc(bb + kk * 2048, C::BOX, 1024), idesc, (cc > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&empty[slot]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) tc::mma_commit(&acc_full[buf]);
            __syncwarp();
        }
        if (lane == 0) {
            s_consumed = it;
            // every MMA issued so far completes before the tensor memory is freed
            tc::mma_commit(&drain);
            tc::mbar_wait(&drain, 0, st);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: running sums of this thread's row and columns, each kept as an
        // unevaluated fp32 pair hi + lo (compensated summation, ~48 significant bits: the exact
        // error of every fp32 addition is carried in lo), much cheaper than float64 arithmetic
        const int lg = warp & 3, half = (warp - 2) >> 2;
        const int f1 = b * 128 + lg * 32 + lane;
        const int f2 = n * TN + half * C::CPT;
        float hi[C::CPT], lo[C::CPT];
        double *srow = state ? state + ((size_t)r * D + f1) * D + f2 : nullptr;
#pragma unroll
        for (int i = 0; i < C::CPT; ++i) {
            const double s0v = srow ? srow[i] : 0.0;
            hi[i] = (float)s0v;
            lo[i] = (float)(s0v - (double)hi[i]);
        }
        const float cf = (float)c;
        bool ok = true, bad = false;
        int seg_i = 0;
        for (int s = s0; s < s1; ++s, ++seg_i) {
            const int buf = seg_i & 1;
            ok = __all_sync(0xffffffffu, tc::mbar_wait(&acc_full[buf], (uint32_t)(seg_i >> 1) & 1u, st));
            if (!ok) break;                            // the TMEM loads below are warp-collective
            tc::fence_after_sync();
            float4 *dst = reinterpret_cast<float4 *>(P + ((size_t)s * D + f1) * D + f2);
#pragma unroll
            for (int q = 0; q < C::CPT / 16; ++q) {
                uint32_t u[16];
                tc::tmem_ld16_nw(tbase + ((uint32_t)(lg * 32) << 16) + (uint32_t)(buf * TN + half * C::CPT + q * 16),
                                 u);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    float pv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = q * 16 + i4 * 4 + e;
                        pv[e] = __fadd_rn(__fmul_rn(cf, hi[i]), __fmul_rn(cf, lo[i]));
                        const float v = __uint_as_float(u[i4 * 4 + e]);
                        bad |= !isfinite(v);
                        // two-sum: hi + v = sum + err exactly
                        const float h = hi[i];
                        const float sum = __fadd_rn(h, v);
                        const float bv = __fsub_rn(sum, h);
                        const float err = __fadd_rn(__fsub_rn(h, __fsub_rn(sum, bv)), __fsub_rn(v, bv));
                        hi[i] = sum;
                        lo[i] = __fadd_rn(lo[i], err);
                    }
                    dst[q * 4 + i4] = make_float4(pv[0], pv[1], pv[2], pv[3]);
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&acc_empty[buf]);
        }
        if (bad) flag(st, DBC_ERR_NONFINITE);
        if (srow && ok) {
#pragma unroll
            for (int i = 0; i < C::CPT; ++i) srow[i] = (double)hi[i] + (double)lo[i];
            if (!diag) {
                // the carried state is the whole symmetric matrix: mirror the off-diagonal block
                double *scol = state + (size_t)r * D * D + f1;
#pragma unroll
                for (int i = 0; i < C::CPT; ++i) scol[(size_t)(f2 + i) * D] = (double)hi[i] + (double)lo[i];
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        // copies still in flight (only after a timeout) land before the CTA leaves
        for (int k = s_consumed; k < issued; ++k) tc::mbar_wait(&full[k % C::NS], (uint32_t)(k / C::NS) & 1u, st);
    }
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tbase, 2 * TN);
}

}  // namespace cr
}  // namespace dbc
