// hnet_route: cosine-similarity boundary router with EMA smoothing.
//
// ByteGen analysis report ("H-Net architecture and its core components";
// "Methodology"): the dynamic chunking module predicts boundaries from the
// cosine similarity of adjacent byte representations and smooths with an
// exponentially weighted average so the discrete choice trains end to end.
// Reading implemented (row vectors):
//   q_t = h_t W_q, k_t = h_t W_k, p_t = 1/2 (1 - cos(q_t, k_{t-1})), p_0 = 1,
//   b_t = [p_t >= threshold]; chunk j of a row starts at the j-th boundary t_j;
//   zbar_j = P_j h_{t_j} + (1 - P_j) zbar_{j-1} with P_j = p_{t_j}.
#include "common.cuh"
#include "gemm_simt.cuh"

namespace dbc {
namespace rt {

struct Layout {
    float *qk;        // [N, 2d]: q in columns [0, d), k in [d, 2d)
    int64_t *count;   // [rows]
    size_t bytes;
};

inline Layout carve(void *ws, int64_t rows, int64_t N, int64_t d) {
    Carver c(ws);
    Layout L;
    L.qk = c.take<float>((size_t)N * 2 * d);
    L.count = c.take<int64_t>(rows + 1);
    L.bytes = c.off;
    return L;
}

__global__ void __launch_bounds__(256) prob_kernel(const float *__restrict__ qk, const int64_t *offsets,
                                                   int64_t rows, int64_t T, int64_t N, int64_t d,
                                                   float threshold, float *p, uint8_t *bnd, int32_t *st) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < N; i += warps) {
        const int64_t r = offsets ? find_row(offsets, rows, i) : i / T;
        int64_t a, n;
        row_bounds(offsets, r, T, a, n);
        float pv = 1.f;
        if (i > a) {
            const float *q = qk + i * 2 * d;
            const float *k = qk + (i - 1) * 2 * d + d;
            float dot = 0.f, nq = 0.f, nk = 0.f;
            for (int64_t j = lane; j < d; j += 32) {
                const float x = q[j], y = k[j];
                dot = fmaf(x, y, dot);
                nq = fmaf(x, x, nq);
                nk = fmaf(y, y, nk);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                dot += __shfl_xor_sync(0xffffffffu, dot, o);
                nq += __shfl_xor_sync(0xffffffffu, nq, o);
                nk += __shfl_xor_sync(0xffffffffu, nk, o);
            }
            const float cs = (nq > 0.f && nk > 0.f) ? dot / (sqrtf(nq) * sqrtf(nk)) : 0.f;
            pv = 0.5f * (1.f - cs);
        }
        if (lane == 0) {
            if (!isfinite(pv)) flag(st, DBC_ERR_NONFINITE);
            p[i] = pv;
            bnd[i] = pv >= threshold ? 1 : 0;
        }
    }
}

__device__ __forceinline__ int64_t block_scan_excl(int64_t v, int64_t *wsum, int64_t *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int64_t w = lane < nw ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    const int64_t r = (wid ? wsum[wid - 1] : 0) + x - v;
    *total = wsum[nw - 1];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(1024) count_kernel(const uint8_t *bnd, const int64_t *offsets,
                                                     int64_t rows, int64_t T, int64_t *count) {
    __shared__ int64_t wsum[32];
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        int64_t a, n;
        row_bounds(offsets, r, T, a, n);
        int64_t c = 0;
        for (int64_t t = threadIdx.x; t < n; t += blockDim.x) c += bnd[a + t];
        int64_t tot;
        block_scan_excl(c, wsum, &tot);
        if (threadIdx.x == 0) count[r] = tot;
    }
}

__global__ void __launch_bounds__(1024) offsets_kernel(const int64_t *count, int64_t rows, int64_t *co) {
    __shared__ int64_t wsum[32];
    __shared__ int64_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int64_t base = 0; base < rows; base += blockDim.x) {
        const int64_t r = base + threadIdx.x;
        const int64_t v = r < rows ? count[r] : 0;
        int64_t tot;
        const int64_t e = block_scan_excl(v, wsum, &tot);
        if (r < rows) co[r] = carry + e;
        __syncthreads();
        if (threadIdx.x == 0) carry += tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) co[rows] = carry;
}

__global__ void __launch_bounds__(1024) compact_kernel(const uint8_t *bnd, const int64_t *offsets,
                                                       int64_t rows, int64_t T, const int64_t *co,
                                                       int64_t *chunk_idx) {
    __shared__ int64_t wsum[32];
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        int64_t a, n;
        row_bounds(offsets, r, T, a, n);
        int64_t carry = co[r];
        for (int64_t base = 0; base < n; base += blockDim.x) {
            const int64_t t = base + threadIdx.x;
            const int64_t f = (t < n) ? bnd[a + t] : 0;
            int64_t tot;
            const int64_t e = block_scan_excl(f, wsum, &tot);
            if (f) chunk_idx[carry + e] = t;
            carry += tot;
        }
    }
}

// One thread per (row, feature): sequential over the row's chunks.
template <class IN>
__global__ void __launch_bounds__(256) ema_kernel(const IN *__restrict__ H, const int64_t *offsets,
                                                  int64_t rows, int64_t T, int64_t d, const float *p,
                                                  const int64_t *co, const int64_t *chunk_idx, float *z) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= rows * d) return;
    const int64_t r = g / d, f = g - (g / d) * d;
    int64_t a, n;
    row_bounds(offsets, r, T, a, n);
    const int64_t c0 = co[r], c1 = co[r + 1];
    float acc = 0.f;
    for (int64_t j = c0; j < c1; ++j) {
        const int64_t t = a + chunk_idx[j];
        const float P = p[t];
        const float x = ld_f(H + t * d + f);
        acc = P * x + (1.f - P) * acc;
        z[j * d + f] = acc;
    }
}

}  // namespace rt
}  // namespace dbc

using namespace dbc;

extern "C" size_t hnet_route_workspace(int64_t rows, int64_t N, int64_t d) {
    if (rows < 0 || N < 0 || d <= 0) return 0;
    return rt::carve(nullptr, rows, N, d).bytes;
}

extern "C" dbc_status hnet_route(const void *H, const int64_t *offsets, int64_t rows, int64_t T,
                                 int64_t N, int64_t d, const void *Wq, const void *Wk, float threshold,
                                 int do_ema, float *p, uint8_t *boundary, int64_t *chunk_idx,
                                 int64_t *chunk_offsets, float *z_smooth, void *ws, size_t ws_bytes,
                                 int32_t *dev_status, dbc_stream_t stream) {
    if (rows < 0 || T < 0 || N < 0 || !isfinite(threshold)) return DBC_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256 && d != 512) return DBC_ERR_UNSUPPORTED;
    if (!offsets && N != rows * T) return DBC_ERR_INVALID_ARG;
    if (!chunk_offsets) return DBC_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0 || rows == 0) {
        if (rows >= 0) cudaMemsetAsync(chunk_offsets, 0, sizeof(int64_t) * (rows + 1), s);
        return launch_status();
    }
    if (!H || !Wq || !Wk || !p || !boundary || !chunk_idx || (do_ema && !z_smooth))
        return DBC_ERR_INVALID_ARG;
    const rt::Layout need = rt::carve(nullptr, rows, N, d);
    if (!ws || ws_bytes < need.bytes || (reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)))
        return DBC_ERR_WORKSPACE;
    const rt::Layout L = rt::carve(ws, rows, N, d);
    const __nv_bfloat16 *Hb = static_cast<const __nv_bfloat16 *>(H);
    dim3 g((unsigned)((N + 63) / 64), (unsigned)(d / 64));
    gemm_bf16_simt<RowIdentity><<<g, 256, 0, s>>>(Hb, d, static_cast<const __nv_bfloat16 *>(Wq), d,
                                                  L.qk, 2 * d, nullptr, 0, N, d, d, RowIdentity{});
    gemm_bf16_simt<RowIdentity><<<g, 256, 0, s>>>(Hb, d, static_cast<const __nv_bfloat16 *>(Wk), d,
                                                  L.qk + d, 2 * d, nullptr, 0, N, d, d, RowIdentity{});
    const int sms = num_sms();
    const int pg = (int)std::max<int64_t>(1, std::min<int64_t>((N + 7) / 8, (int64_t)sms * 32));
    rt::prob_kernel<<<pg, 256, 0, s>>>(L.qk, offsets, rows, T, N, d, threshold, p, boundary, dev_status);
    const int rg = (int)std::min<int64_t>(rows, 65535);
    rt::count_kernel<<<rg, 1024, 0, s>>>(boundary, offsets, rows, T, L.count);
    rt::offsets_kernel<<<1, 1024, 0, s>>>(L.count, rows, chunk_offsets);
    rt::compact_kernel<<<rg, 1024, 0, s>>>(boundary, offsets, rows, T, chunk_offsets, chunk_idx);
    count_launches(do_ema ? 7 : 6);
    if (do_ema) {
        const int64_t th = rows * d;
        rt::ema_kernel<__nv_bfloat16><<<(unsigned)((th + 255) / 256), 256, 0, s>>>(
            Hb, offsets, rows, T, d, p, chunk_offsets, chunk_idx, z_smooth);
    }
    return launch_status();
}
