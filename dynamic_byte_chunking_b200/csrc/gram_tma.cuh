// Segment Grams G_s = X_s^T X_s (d = 256, bf16 x bf16 exact, fp32 accumulation in TMEM), one CTA per
// segment, for the segment-parallel P path: only the blocks the factor kernel reads (the first 128
// rows' first 128 columns, and all columns of the last 128 rows).
//   * one thread streams the segment's positions with TMA (boxes of 64 positions x 64 features,
//     128-byte swizzle, tensor map over this GPU's own memory, no multicast) through a 4-stage ring
//     and issues the MMAs (both operands MN-major, positions are K); positions past the segment's
//     end inside its last 16-position step are zeroed in shared memory first;
//   * the accumulators go to shared memory as 128 x 32 fp32 tiles in the 128-byte swizzled layout
//     and leave with TMA tile stores, so the global writes are whole lines.
// Every wait is bounded; a timeout flags DBC_ERR_TIMEOUT and the CTA skips its remaining work.
#pragma once

#include <cuda.h>

#include "tc.cuh"

namespace dbc {
namespace cr {

struct GramTma {
    static constexpr int D = 256;
    static constexpr int KC = 64;                          // positions per stage
    static constexpr int NS = 4;
    static constexpr uint32_t BOX = 64 * 128;              // 64 positions x 64 features, bf16
    static constexpr uint32_t STAGE = 4 * BOX;             // all 256 features
    static constexpr uint32_t TILE = 128 * 128;            // 128 rows x 32 fp32 columns
    static constexpr int NTILE = 4 + 8;                    // first row block: 4 column tiles, second: 8
    static constexpr size_t SMEM = (NTILE * TILE > NS * STAGE ? NTILE * TILE : NS * STAGE) + 1024;
};

__global__ void __launch_bounds__(256, 1) gram_tma_kernel(const __grid_constant__ CUtensorMap tmH,
                                                          const __grid_constant__ CUtensorMap tmG, Segs S,
                                                          int32_t *st) {
    using C = GramTma;
    constexpr int D = C::D;
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t full[C::NS], empty[C::NS], done;
    __shared__ uint32_t tmem_base;
    __shared__ int s_ok;
    const int s = blockIdx.x;
    if (s >= *S.nseg) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int len = S.len[s];
    const int64_t start = S.start[s];
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    uint8_t *const sgen = smraw + (base - tc::smem_u32(smraw));
    if (warp == 0) tc::tmem_alloc(&tmem_base, 512);
    if (tid == 0) {
        for (int i = 0; i < C::NS; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        tc::mbar_init(&done, 1);
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmH);
        tc::tma_prefetch_desc(&tmG);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const int nchunks = (len + C::KC - 1) / C::KC;

    if (tid == 0) {
        bool ok = true;
        auto load = [&](int c) {
            const int slot = c % C::NS;
            const uint32_t sb = base + (uint32_t)slot * C::STAGE;
            tc::mbar_arrive_expect_tx(&full[slot], C::STAGE);
            for (int q = 0; q < 4; ++q)
                tc::tma_load_2d(sb + (uint32_t)q * C::BOX, &tmH, &full[slot], q * 64, (int)(start + c * C::KC));
        };
        for (int c = 0; c < C::NS - 1 && c < nchunks; ++c) load(c);
        constexpr uint32_t id256 = tc::idesc_bf16(128, 256, true, true);
        constexpr uint32_t id128 = tc::idesc_bf16(128, 128, true, true);
        int issued = min(C::NS - 1, nchunks);
        for (int c = 0; c < nchunks && ok; ++c) {
            const int cn = c + C::NS - 1;
            if (cn < nchunks) {
                if (cn >= C::NS) ok = tc::mbar_wait(&empty[cn % C::NS], (uint32_t)((cn / C::NS) - 1) & 1u, st);
                if (!ok) break;
                load(cn);
                issued = cn + 1;
            }
            const int slot = c % C::NS;
            ok = tc::mbar_wait(&full[slot], (uint32_t)(c / C::NS) & 1u, st);
            if (!ok) break;
            const uint32_t sb = base + (uint32_t)slot * C::STAGE;
            const int valid = min(C::KC, len - c * C::KC);
            const int ksteps = (valid + 15) >> 4;
            if (valid & 15) {
                // positions past the segment end inside the last K step read as zero rows
                for (int q = 0; q < 4; ++q)
                    for (int r = valid; r < ksteps * 16; ++r)
                        for (int ch = 0; ch < 8; ++ch)
                            asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(
                                             sb + (uint32_t)q * C::BOX + (uint32_t)r * 128 + ch * 16),
                                         "r"(0)
                                         : "memory");
                tc::fence_async_smem();
            }
            tc::fence_after_sync();
            for (int kk = 0; kk < ksteps; ++kk) {
                // rows 0..127 x columns 0..127, rows 128..255 x columns 0..255
                tc::mma_bf16(tbase, tc::sdesc(sb + kk * 2048, C::BOX, 1024), tc::sdesc(sb + kk * 2048, C::BOX, 1024),
                             id128, (c > 0 || kk > 0) ? 1u : 0u);
                tc::mma_bf16(tbase + 256u, tc::sdesc(sb + 2 * C::BOX + kk * 2048, C::BOX, 1024),
                             tc::sdesc(sb + kk * 2048, C::BOX, 1024), id256, (c > 0 || kk > 0) ? 1u : 0u);
            }
            tc::mma_commit(&empty[slot]);
        }
        // every MMA issued lands (and with it every copy it read) before the epilogue reuses the stages
        tc::mma_commit(&done);
        if (!tc::mbar_wait(&done, 0, st)) ok = false;
        // copies issued but never consumed (only after a timeout) land before the CTA reuses smem
        for (int k = 0; k < issued; ++k)
            if (!ok) tc::mbar_wait(&full[k % C::NS], (uint32_t)(k / C::NS) & 1u, st);
        s_ok = ok ? 1 : 0;
    }
    __syncthreads();
    tc::fence_after_sync();
    const bool ok = s_ok != 0;
    bool bad = false;
    if (ok) {
        // warp w: TMEM lanes (w % 4) * 32 .. + 31, row block m = w / 4 (rows m*128 + ..), its tiles
        const int lg = warp & 3, m = warp >> 2;
        const int r = lg * 32 + lane;                          // row inside the block
        const int ncols = m == 0 ? 128 : 256;
        const int tile0 = m == 0 ? 0 : 4;
        for (int t = 0; t < ncols / 32; ++t) {
            uint32_t u[2][16];
            const uint32_t ta = tbase + ((uint32_t)(lg * 32) << 16) + (uint32_t)(m * 256 + t * 32);
            tc::tmem_ld16_nw(ta, u[0]);
            tc::tmem_ld16_nw(ta + 16, u[1]);
            tc::tmem_wait_ld();
            const int grow = m * 128 + r;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (grow == t * 32 + i) bad |= !isfinite(__uint_as_float(u[i >> 4][i & 15]));
            uint8_t *tile = sgen + (size_t)(tile0 + t) * C::TILE;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t *x = &u[ch >> 2][(ch & 3) * 4];
                *reinterpret_cast<uint4 *>(tile + r * 128 + ((ch ^ (r & 7)) * 16)) = make_uint4(x[0], x[1], x[2], x[3]);
            }
        }
        tc::fence_async_smem();
    }
    if (bad) flag(st, DBC_ERR_NONFINITE);
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
        const int y0 = s * D;
        for (int t = 0; t < C::NTILE; ++t) {
            const int m = t < 4 ? 0 : 1, tc_ = t < 4 ? t : t - 4;
            const uint32_t src = base + (uint32_t)t * C::TILE;
            asm volatile(
                "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(&tmG),
                "r"(tc_ * 32), "r"(y0 + m * 128), "r"(src)
                : "memory");
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        // shared memory must outlive the stores' reads of it; the writes complete with the kernel
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

}  // namespace cr
}  // namespace dbc
