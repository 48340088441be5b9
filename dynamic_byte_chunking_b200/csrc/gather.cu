// chunk_gather: z_k = h_{s_k} for every boundary (ByteFlow, paper.rainbus.top
// summary, "Method steps", stage 2), optionally followed by z_k W_proj.
//
// The copy is bit-exact: one warp per chunk row moves the row with 16-byte
// vector loads/stores.  The projection is a bf16 GEMM with fp32 accumulation.
#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"

namespace dbc {
namespace ga {

__global__ void __launch_bounds__(256) gather_kernel(const uint4 *__restrict__ H, const int64_t *offsets,
                                                     int64_t T, int64_t vec_per_row,
                                                     const int64_t *__restrict__ idx,
                                                     const int64_t *__restrict__ idx_offsets, int64_t rows,
                                                     int64_t total, uint4 *__restrict__ Z, int32_t *st) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t k = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); k < total; k += warps) {
        const int64_t r = find_row(idx_offsets, rows, k);
        int64_t a, n;
        row_bounds(offsets, r, T, a, n);
        const int64_t t = idx[k];
        uint4 *dst = Z + k * vec_per_row;
        if (t < 0 || t >= n) {
            if (lane == 0) flag(st, DBC_ERR_BOUNDS);
            for (int64_t v = lane; v < vec_per_row; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
            continue;
        }
        const uint4 *src = H + (a + t) * vec_per_row;
        for (int64_t v = lane; v < vec_per_row; v += 32) dst[v] = src[v];
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
    const int64_t want = (total_K + 7) / 8;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 16));
    ga::gather_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4 *>(H), offsets, T, vpr, idx,
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
