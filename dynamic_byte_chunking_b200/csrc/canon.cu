// canon_conv1d: the Canon layer of the local encoder, a causal depthwise
// convolution with kernel 4 (ByteFlow notes, "Key design 1"; summary, "Method
// steps", stage 1: SWA + Canon(causal_conv1d, k = 4) + SwiGLU), whose output
// feeds the coding-rate chunker; chunk_coding_rate_canon runs it and the
// chunker in one call.
//
//   out_t[f] = bf16( bias[f] (+ h_t[f]) + sum_{j=0..3} w[f, j] h_{t-j}[f] ),
//   h before a row's first position = 0, each row of a packed batch alone.
//
// Arithmetic: fp32, in the fixed order bias, residual, tap 0, 1, 2, 3 (every
// product of two bf16 values is exact in fp32, each fma rounds once), then one
// round-to-nearest-even to bf16.  HBM-bound: one warp walks a block of
// consecutive positions of a row, lane g holding features 8g .. 8g+7 and the
// last three inputs in registers, so H is read once and written once with
// 16-byte accesses.
#include "common.cuh"

namespace dbc {
namespace cv {

constexpr int kThreads = 256;
constexpr int kPos = 32;            // positions per warp

// One lane: 8 features of one position.
struct Vec8 {
    float v[8];
};

__device__ __forceinline__ Vec8 unpack(uint4 u) {
    Vec8 r;
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        r.v[2 * i] = __uint_as_float(w[i] << 16);
        r.v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    return r;
}

__device__ __forceinline__ uint4 pack(const float (&a)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(a[2 * i]));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(a[2 * i + 1]));
        w[i] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Row containing position t (offsets non-decreasing, offsets[0] = 0).
__device__ __forceinline__ int64_t row_of(const int64_t *offsets, int64_t rows, int64_t t) {
    int64_t lo = 0, hi = rows;
    while (hi - lo > 1) {
        const int64_t mid = (lo + hi) >> 1;
        if (offsets[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kThreads) canon_kernel(const uint4 *__restrict__ H, const int64_t *offsets,
                                                         int64_t rows, int64_t T, int64_t N, int d8,
                                                         const __nv_bfloat16 *__restrict__ w,
                                                         const __nv_bfloat16 *__restrict__ bias, int residual,
                                                         uint4 *__restrict__ out, int32_t *st) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t nblk = (N + kPos - 1) / kPos;
    for (int g = lane; g < d8; g += 32) {
        float wk[4][8], bv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int f = g * 8 + i;
#pragma unroll
            for (int j = 0; j < 4; ++j) wk[j][i] = __bfloat162float(w[f * 4 + j]);
            bv[i] = bias ? __bfloat162float(bias[f]) : 0.f;
        }
        for (int64_t blk = warp; blk < nblk; blk += nwarps) {
            const int64_t p0 = blk * kPos, p1 = min(N, p0 + kPos);
            int64_t r = offsets ? row_of(offsets, rows, p0) : p0 / T;
            int64_t rs = offsets ? offsets[r] : r * T;
            int64_t re = offsets ? offsets[r + 1] : rs + T;
            if (p0 < rs || p0 >= re) {          // malformed offsets
                if (g == lane && lane == 0) flag(st, DBC_ERR_BOUNDS);
                break;
            }
            Vec8 h1 = {}, h2 = {}, h3 = {};
            if (p0 - 1 >= rs) h1 = unpack(H[(p0 - 1) * d8 + g]);
            if (p0 - 2 >= rs) h2 = unpack(H[(p0 - 2) * d8 + g]);
            if (p0 - 3 >= rs) h3 = unpack(H[(p0 - 3) * d8 + g]);
            auto step = [&](const Vec8 &h0, int64_t t) {
                float o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float acc = bv[i];
                    if (residual) acc = __fadd_rn(acc, h0.v[i]);
                    acc = fmaf(wk[0][i], h0.v[i], acc);
                    acc = fmaf(wk[1][i], h1.v[i], acc);
                    acc = fmaf(wk[2][i], h2.v[i], acc);
                    acc = fmaf(wk[3][i], h3.v[i], acc);
                    o[i] = acc;
                }
                out[t * d8 + g] = pack(o);
                h3 = h2;
                h2 = h1;
                h1 = h0;
            };
            int64_t t = p0;
            while (t < p1) {
                while (t >= re && r + 1 < rows) {   // next row: the window restarts from zeros
                    ++r;
                    rs = re;
                    re = offsets ? offsets[r + 1] : rs + T;
                    h1 = Vec8{};
                    h2 = Vec8{};
                    h3 = Vec8{};
                }
                if (t + 4 <= p1 && t + 4 <= re) {
                    // four positions of one row: all loads in flight before the arithmetic
                    uint4 u[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) u[q] = H[(t + q) * d8 + g];
#pragma unroll
                    for (int q = 0; q < 4; ++q) step(unpack(u[q]), t + q);
                    t += 4;
                } else {
                    step(unpack(H[t * d8 + g]), t);
                    ++t;
                }
            }
        }
    }
}

}  // namespace cv
}  // namespace dbc

using namespace dbc;

static dbc_status canon_args(const void *H, const int64_t *offsets, int64_t rows, int64_t T, int64_t N, int64_t d,
                             const void *w, const void *out) {
    if (rows < 0 || T < 0 || N < 0 || d <= 0) return DBC_ERR_INVALID_ARG;
    if (d % 8 || d > 4096) return DBC_ERR_UNSUPPORTED;
    if (!offsets && N != rows * T) return DBC_ERR_INVALID_ARG;
    if (N == 0 || rows == 0) return DBC_OK;
    if (!H || !w || !out || !aligned16(H) || !aligned16(out)) return DBC_ERR_INVALID_ARG;
    return DBC_OK;
}

static dbc_status launch_canon(const void *H, const int64_t *offsets, int64_t rows, int64_t T, int64_t N, int64_t d,
                               const void *w, const void *bias, int residual, void *out, int32_t *dev_status,
                               cudaStream_t s) {
    const int64_t nblk = (N + cv::kPos - 1) / cv::kPos;
    const int64_t want = (nblk + cv::kThreads / 32 - 1) / (cv::kThreads / 32);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)num_sms() * 16));
    cv::canon_kernel<<<grid, cv::kThreads, 0, s>>>(static_cast<const uint4 *>(H), offsets, rows, T, N, (int)(d / 8),
                                                   static_cast<const __nv_bfloat16 *>(w),
                                                   static_cast<const __nv_bfloat16 *>(bias), residual ? 1 : 0,
                                                   static_cast<uint4 *>(out), dev_status);
    count_launches(1);
    return launch_status();
}

extern "C" dbc_status canon_conv1d(const void *H, const int64_t *offsets, int64_t rows, int64_t T, int64_t N,
                                   int64_t d, const void *w, const void *bias, int residual, void *out,
                                   int32_t *dev_status, dbc_stream_t stream) {
    DBC_NVTX_RANGE("canon_conv1d");
    const dbc_status a = canon_args(H, offsets, rows, T, N, d, w, out);
    if (a != DBC_OK || N == 0 || rows == 0) return a;
    return launch_canon(H, offsets, rows, T, N, d, w, bias, residual, out, dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}

extern "C" dbc_status chunk_coding_rate_canon(const void *H, const int64_t *offsets, int64_t rows, int64_t T,
                                              int64_t N, int64_t d, const void *w, const void *bias, int residual,
                                              void *Hc, float eps2, float *dR, void *ws, size_t ws_bytes,
                                              int32_t *dev_status, dbc_stream_t stream) {
    DBC_NVTX_RANGE("chunk_coding_rate_canon");
    const dbc_status a = canon_args(H, offsets, rows, T, N, d, w, Hc);
    if (a != DBC_OK) return a;
    if (!(eps2 > 0.f) || !std::isfinite(eps2)) return DBC_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256 && d != 512) return DBC_ERR_UNSUPPORTED;
    if (N == 0 || rows == 0) return DBC_OK;
    if (!dR) return DBC_ERR_INVALID_ARG;
    if (!ws || ws_bytes < chunk_coding_rate_workspace(rows, T, N, d)) return DBC_ERR_WORKSPACE;
    const dbc_status c = launch_canon(H, offsets, rows, T, N, d, w, bias, residual, Hc, dev_status,
                                      reinterpret_cast<cudaStream_t>(stream));
    if (c != DBC_OK) return c;
    return chunk_coding_rate(Hc, DBC_BF16, offsets, rows, T, N, d, eps2, dR, ws, ws_bytes, dev_status, stream);
}
