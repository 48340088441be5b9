// C[M, N] = A[M, K] B[K, N] on tcgen05: A row-major bf16 (K-major operand),
// B row-major bf16 [K][N] (read as an MN-major operand), fp32 accumulation in
// TMEM.  One CTA = 128 rows x up to 256 columns; K in 64-deep chunks, three
// cp.async stages; epilogue writes fp32 and/or bf16 (round to nearest even).
// Requires K % 64 == 0, N % 64 == 0, 16-byte aligned rows.
#pragma once

#include "tc.cuh"

namespace dbc {
namespace gt {

struct Cfg {
    static constexpr int NS = 3;
    static constexpr uint32_t A_BYTES = 128 * 128;
    static constexpr uint32_t B_BYTES = 4 * 64 * 128;
    static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
    static constexpr size_t SMEM = NS * STAGE + 1024;
};

__global__ void __launch_bounds__(128, 1) gemm_tc_kernel(const __nv_bfloat16 *__restrict__ A, int64_t lda,
                                                         const __nv_bfloat16 *__restrict__ B, int64_t ldb,
                                                         float *C, int64_t ldc, __nv_bfloat16 *Cb, int64_t ldcb,
                                                         int64_t M, int64_t N, int64_t K, int32_t *st) {
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[Cfg::NS];
    __shared__ uint32_t tmem_base;
    const int64_t m0 = (int64_t)blockIdx.x * 128, n0 = (int64_t)blockIdx.y * 256;
    if (m0 >= M || n0 >= N) return;
    const int nt = (int)(N - n0 < 256 ? N - n0 : 256);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
    if (tid == 0) {
        for (int i = 0; i < Cfg::NS; ++i) tc::mbar_init(&mbar[i], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const int nchunks = (int)(K / 64), nb8 = nt / 8;
    auto load = [&](int c, uint32_t sa) {
        for (int e = tid; e < 128 * 8; e += 128) {
            const int r = e >> 3, ch = e & 7;
            const bool in = m0 + r < M;
            tc::cp_async16(sa + tc::kmajor_off(r, ch * 8), A + (in ? m0 + r : 0) * lda + c * 64 + ch * 8,
                           in ? 16u : 0u);
        }
        const uint32_t sb = sa + Cfg::A_BYTES;
        for (int e = tid; e < 64 * nb8; e += 128) {
            const int k = e / nb8, n8 = e - (e / nb8) * nb8;
            tc::cp_async16(sb + tc::mnmajor_off(n8 * 8, k, 8192), B + (size_t)(c * 64 + k) * ldb + n0 + n8 * 8, 16u);
        }
    };
    const uint32_t idesc = tc::idesc_bf16(128, nt, false, true);
    bool ok = true;
    for (int c = 0; c < Cfg::NS - 1; ++c) {
        if (c < nchunks) load(c, base + (uint32_t)c * Cfg::STAGE);
        tc::cp_async_commit();
    }
    for (int c = 0; c < nchunks; ++c) {
        const int cn = c + Cfg::NS - 1;
        if (cn < nchunks) {
            if (cn >= Cfg::NS) ok &= tc::mbar_wait(&mbar[cn % Cfg::NS], (uint32_t)((cn / Cfg::NS) - 1) & 1u, st);
            load(cn, base + (uint32_t)(cn % Cfg::NS) * Cfg::STAGE);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<Cfg::NS - 1>();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t sa = base + (uint32_t)(c % Cfg::NS) * Cfg::STAGE, sb = sa + Cfg::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tbase, tc::sdesc(sa + kk * 32, 16, 1024), tc::sdesc(sb + kk * 2048, 8192, 1024), idesc,
                             (c > 0 || kk > 0) ? 1u : 0u);
            tc::mma_commit(&mbar[c % Cfg::NS]);
        }
        __syncthreads();
    }
    if (nchunks > 0) ok &= tc::mbar_wait(&mbar[(nchunks - 1) % Cfg::NS], (uint32_t)((nchunks - 1) / Cfg::NS) & 1u, st);
    ok = __syncthreads_and(ok) != 0;
    tc::fence_after_sync();
    if (ok) {
        const int64_t row = m0 + warp * 32 + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < nt; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
            if (row < M) {
                if (C) {
                    float4 *d = reinterpret_cast<float4 *>(C + row * ldc + n0 + c0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
                if (Cb) {
                    __align__(16) __nv_bfloat16 h[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) h[i] = __float2bfloat16_rn(v[i]);
                    uint4 *d = reinterpret_cast<uint4 *>(Cb + row * ldcb + n0 + c0);
                    d[0] = reinterpret_cast<uint4 *>(h)[0];
                    d[1] = reinterpret_cast<uint4 *>(h)[1];
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}

inline void launch_gemm_tc(const __nv_bfloat16 *A, int64_t lda, const __nv_bfloat16 *B, int64_t ldb, float *C,
                           int64_t ldc, __nv_bfloat16 *Cb, int64_t ldcb, int64_t M, int64_t N, int64_t K,
                           int32_t *st, cudaStream_t s) {
    cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
    dim3 g((unsigned)((M + 127) / 128), (unsigned)((N + 255) / 256));
    gemm_tc_kernel<<<g, 128, Cfg::SMEM, s>>>(A, lda, B, ldb, C, ldc, Cb, ldcb, M, N, K, st);
}

}  // namespace gt
}  // namespace dbc
