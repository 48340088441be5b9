// Plain CUDA-core bf16 x bf16 -> fp32 tile GEMM used by the first versions of
// the projection and router kernels: C[M, N] = A[M, K] B[K, N], row-major,
// 64 x 64 tiles, 32-deep K steps, 4 x 4 outputs per thread.
#pragma once

#include "common.cuh"

namespace dbc {

// Optional A-row indirection: row i of the logical A is A[arow(i)].
struct RowIdentity {
    __device__ __forceinline__ int64_t operator()(int64_t i) const { return i; }
};

template <class ARow>
__global__ void __launch_bounds__(256) gemm_bf16_simt(const __nv_bfloat16 *__restrict__ A, int64_t lda,
                                                      const __nv_bfloat16 *__restrict__ B, int64_t ldb,
                                                      float *C, int64_t ldc, __nv_bfloat16 *Cb, int64_t ldcb,
                                                      int64_t M, int64_t N, int64_t K, ARow arow) {
    __shared__ float As[32][65];
    __shared__ float Bs[32][64];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int64_t m0 = (int64_t)blockIdx.x * 64, n0 = (int64_t)blockIdx.y * 64;
    float acc[4][4] = {};
    for (int64_t k0 = 0; k0 < K; k0 += 32) {
        for (int e = tid; e < 64 * 32; e += 256) {
            const int rr = e >> 5, kk = e & 31;
            const int64_t i = m0 + rr;
            As[kk][rr] = (i < M && k0 + kk < K) ? __bfloat162float(A[arow(i) * lda + k0 + kk]) : 0.f;
        }
        for (int e = tid; e < 32 * 64; e += 256) {
            const int kk = e >> 6, cc = e & 63;
            Bs[kk][cc] = (k0 + kk < K && n0 + cc < N) ? __bfloat162float(B[(k0 + kk) * ldb + n0 + cc]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) { a[q] = As[kk][ty * 4 + q]; b[q] = Bs[kk][tx * 4 + q]; }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[q][r] = fmaf(a[q], b[r], acc[q][r]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int64_t i = m0 + ty * 4 + q;
        if (i >= M) continue;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t j = n0 + tx * 4 + r;
            if (j >= N) continue;
            if (C) C[i * ldc + j] = acc[q][r];
            if (Cb) Cb[i * ldcb + j] = __float2bfloat16_rn(acc[q][r]);
        }
    }
}

}  // namespace dbc
