// chunk_gather: z_k = h_{s_k} for every boundary (ByteFlow, paper.rainbus.top
// summary, "Method steps", stage 2), optionally followed by z_k W_proj.
//
// The copy is bit-exact: 16-byte vector loads/stores, several rows per warp
// in flight.  The projection is a bf16 GEMM with fp32 accumulation.
#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"

namespace dbc {
namespace ga {

constexpr int kGatherThreads = 256;
constexpr int kRowsPerWarp = 4;         // chunk rows one warp moves per step (loads in flight together)
constexpr int kOffsCache = 4096;        // idx_offsets entries cached in shared memory

// One warp moves kRowsPerWarp chunk rows per step: lanes 0..3 look up the rows'
// sources (row of the chunk by binary search over idx_offsets, cached in shared
// memory when it fits, and the boundary index), the warp then issues every
// 16-byte load of those rows before the stores.
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const uint4 *__restrict__ H, const int64_t *offsets,
                                                                int64_t T, int64_t vec_per_row,
                                                                const int64_t *__restrict__ idx,
                                                                const int64_t *__restrict__ idx_offsets, int64_t rows,
                                                                int64_t total, uint4 *__restrict__ Z, int32_t *st) {
    __shared__ int64_t s_offs[kOffsCache];
    const bool cached = rows + 1 <= kOffsCache;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kGatherThreads / 32);
    const int64_t k_first = ((int64_t)blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5)) * kRowsPerWarp;
    // the first step's boundary index is loaded together with the offsets cache (it does not
    // depend on the row)
    int64_t t_next = lane < kRowsPerWarp && k_first + lane < total ? idx[k_first + lane] : 0;
    if (cached)
        for (int64_t i = threadIdx.x; i <= rows; i += blockDim.x) s_offs[i] = idx_offsets[i];
    __syncthreads();
    const int64_t *offs = cached ? s_offs : idx_offsets;
    for (int64_t k0 = k_first; k0 < total; k0 += warps * kRowsPerWarp) {
        // source row start (in vectors) of chunk k0 + lane, or -1 (out of range / bad index)
        int64_t src = -1;
        const int64_t t = t_next;
        const int64_t kn = k0 + warps * kRowsPerWarp + lane;
        if (lane < kRowsPerWarp && kn < total) t_next = idx[kn];
        if (lane < kRowsPerWarp && k0 + lane < total) {
            const int64_t k = k0 + lane;
            const int64_t r = find_row(offs, rows, k);
            int64_t a, n;
            row_bounds(offsets, r, T, a, n);
            if (t < 0 || t >= n) flag(st, DBC_ERR_BOUNDS);
            else src = (a + t) * vec_per_row;
        }
        int64_t srcs[kRowsPerWarp];
#pragma unroll
        for (int q = 0; q < kRowsPerWarp; ++q) srcs[q] = __shfl_sync(0xffffffffu, src, q);
        for (int64_t v = lane; v < vec_per_row; v += 32) {
            uint4 val[kRowsPerWarp];
#pragma unroll
            for (int q = 0; q < kRowsPerWarp; ++q)
                val[q] = srcs[q] >= 0 ? H[srcs[q] + v] : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < kRowsPerWarp; ++q)
                if (k0 + q < total) Z[(k0 + q) * vec_per_row + v] = val[q];
        }
    }
}

}  // namespace ga
}  // namespace dbc

using namespace dbc;

extern "C" dbc_status chunk_gather(const void *H, int dtype, const int64_t *offsets, int64_t T,
                                   int64_t d, const int64_t *idx, const int64_t *idx_offsets,
                                   int64_t rows, int64_t total_K, void *Z, const void *W_proj,
                                   int64_t d_g, float *Zp_f32, void *Zp_bf16, int32_t *dev_status,
                                   dbc_stream_t stream) {
    DBC_NVTX_RANGE("chunk_gather");
    if (rows < 0 || T < 0 || total_K < 0 || d <= 0) return DBC_ERR_INVALID_ARG;
    if (dtype != DBC_F32 && dtype != DBC_BF16) return DBC_ERR_UNSUPPORTED;
    const int64_t esz = dtype == DBC_BF16 ? 2 : 4;
    if ((d * esz) % 16) return DBC_ERR_UNSUPPORTED;
    if (total_K == 0 || rows == 0) return DBC_OK;
    if (!H || !idx || !idx_offsets || !Z || !aligned16(H) || !aligned16(Z)) return DBC_ERR_INVALID_ARG;
    if (W_proj) {
        if (dtype != DBC_BF16 || d_g <= 0 || d % 32 || (!Zp_f32 && !Zp_bf16)) return DBC_ERR_INVALID_ARG;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t vpr = d * esz / 16;
    const int sms = num_sms();
    const int64_t per_cta = (ga::kGatherThreads / 32) * ga::kRowsPerWarp;
    const int64_t want = (total_K + per_cta - 1) / per_cta;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8));
    ga::gather_kernel<<<grid, ga::kGatherThreads, 0, s>>>(static_cast<const uint4 *>(H), offsets, T, vpr, idx,
                                           idx_offsets, rows, total_K, static_cast<uint4 *>(Z),
                                           dev_status);
    count_launches(W_proj ? 2 : 1);
    if (W_proj) {
        const __nv_bfloat16 *Zb = static_cast<const __nv_bfloat16 *>(Z);
        const __nv_bfloat16 *Wp = static_cast<const __nv_bfloat16 *>(W_proj);
        if (d % 64 == 0 && d_g % 64 == 0) {
            gt::launch_gemm_tc(Zb, d, Wp, d_g, Zp_f32, d_g, static_cast<__nv_bfloat16 *>(Zp_bf16), d_g, total_K, d_g,
                               d, dev_status, s);
        } else {
            dim3 g((unsigned)((total_K + 63) / 64), (unsigned)((d_g + 63) / 64));
            gemm_bf16_simt<RowIdentity><<<g, 256, 0, s>>>(Zb, d, Wp, d_g, Zp_f32, d_g,
                                                          static_cast<__nv_bfloat16 *>(Zp_bf16), d_g, total_K, d_g,
                                                          d, RowIdentity{});
        }
    }
    return launch_status();
}
