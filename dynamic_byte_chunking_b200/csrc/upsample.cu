// chunk_upsample: multi-linear upsampling with residual.
//
// ByteFlow (paper.rainbus.top summary, "Method steps", stage 4; papernotes.org
// notes, "Key design 4"): each position t belongs to chunk c(t), the last
// boundary s_c <= t; it falls into one of B bins with its own matrix W_b, and
// S_t = h_t + g_{c(t)} W_{b(t)}.
//
// Positions are classified (chunk, bin), counted per bin and permuted so that
// each bin's positions are contiguous; the product is then a grouped GEMM over
// bins whose A rows are gathered chunk vectors and whose output rows are
// scattered back to their positions with the residual added.
#include "common.cuh"

namespace dbc {
namespace up {

constexpr int kMaxBins = 64;

struct Layout {
    int32_t *chunk;      // [N] global chunk row of each position
    uint8_t *bin;        // [N]
    int32_t *perm;       // [N] positions grouped by bin
    int32_t *hist;       // [kMaxBins]
    int32_t *cursor;     // [kMaxBins]
    int32_t *bin_start;  // [kMaxBins + 1]
    int32_t *tile_start; // [kMaxBins + 1]
    size_t bytes;
};

inline Layout carve(void *ws, int64_t N) {
    Carver c(ws);
    Layout L;
    L.chunk = c.take<int32_t>(N + 1);
    L.bin = c.take<uint8_t>(N + 1);
    L.perm = c.take<int32_t>(N + 1);
    L.hist = c.take<int32_t>(kMaxBins);
    L.cursor = c.take<int32_t>(kMaxBins);
    L.bin_start = c.take<int32_t>(kMaxBins + 1);
    L.tile_start = c.take<int32_t>(kMaxBins + 1);
    L.bytes = c.off;
    return L;
}

__global__ void __launch_bounds__(256) classify_kernel(const int64_t *offsets, int64_t T, int64_t N,
                                                       const int64_t *__restrict__ idx,
                                                       const int64_t *__restrict__ idx_offsets, int64_t rows,
                                                       int nbins, int mode, Layout L, int32_t *st) {
    __shared__ int32_t h[kMaxBins];
    for (int b = threadIdx.x; b < nbins; b += blockDim.x) h[b] = 0;
    __syncthreads();
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < N;
         p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = offsets ? find_row(offsets, rows, p) : p / T;
        int64_t a, n;
        row_bounds(offsets, r, T, a, n);
        const int64_t t = p - a;
        const int64_t ia = idx_offsets[r];
        const int64_t kr = idx_offsets[r + 1] - ia;
        int64_t c = 0;
        if (kr <= 0 || idx[ia] != 0) {
            flag(st, DBC_ERR_BOUNDS);
        } else {
            int64_t lo = 0, hi = kr;     // idx[ia+lo] <= t < idx[ia+hi] (hi = kr: +inf)
            while (hi - lo > 1) {
                const int64_t mid = (lo + hi) >> 1;
                if (idx[ia + mid] <= t) lo = mid; else hi = mid;
            }
            c = lo;
        }
        const int64_t sc = kr > 0 ? idx[ia + c] : 0;
        int64_t b;
        if (mode == DBC_BIN_IN_CHUNK_OFFSET) {
            b = t - sc;
            if (b > nbins - 1) b = nbins - 1;
        } else if (mode == DBC_BIN_IN_CHUNK_FRACTION) {
            const int64_t nxt = (c + 1 < kr) ? idx[ia + c + 1] : n;
            const int64_t len = nxt - sc;
            b = len > 0 ? ((int64_t)nbins * (t - sc)) / len : 0;
        } else {
            b = ((int64_t)t * nbins) / n;
        }
        if (b < 0 || b >= nbins) {
            flag(st, DBC_ERR_BOUNDS);
            b = b < 0 ? 0 : nbins - 1;
        }
        L.chunk[p] = (int32_t)(ia + c);
        L.bin[p] = (uint8_t)b;
        atomicAdd(&h[b], 1);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < nbins; b += blockDim.x)
        if (h[b]) atomicAdd(&L.hist[b], h[b]);
}

__global__ void scan_bins_kernel(int nbins, Layout L) {
    if (threadIdx.x == 0) {
        int32_t s = 0, t = 0;
        for (int b = 0; b < nbins; ++b) {
            L.bin_start[b] = s;
            L.tile_start[b] = t;
            L.cursor[b] = 0;
            s += L.hist[b];
            t += (L.hist[b] + 63) / 64;
        }
        L.bin_start[nbins] = s;
        L.tile_start[nbins] = t;
    }
}

__global__ void __launch_bounds__(256) scatter_kernel(int64_t N, Layout L) {
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < N;
         p += (int64_t)gridDim.x * blockDim.x) {
        const int b = L.bin[p];
        const int slot = atomicAdd(&L.cursor[b], 1);
        L.perm[L.bin_start[b] + slot] = (int32_t)p;
    }
}

// Grouped GEMM tile: 64 positions of one bin x 64 output columns.
template <class IN>
__global__ void __launch_bounds__(256) bin_gemm_kernel(const __nv_bfloat16 *__restrict__ G, int64_t dg,
                                                       const IN *__restrict__ H, int64_t dl,
                                                       const __nv_bfloat16 *__restrict__ W, int nbins,
                                                       Layout L, float *__restrict__ S) {
    const int tile = blockIdx.x;
    if (tile >= L.tile_start[nbins]) return;
    int b = 0;
    while (b + 1 < nbins && L.tile_start[b + 1] <= tile) ++b;
    const int r0 = L.bin_start[b] + (tile - L.tile_start[b]) * 64;
    const int cnt = min(64, L.bin_start[b + 1] - r0);
    const int64_t n0 = (int64_t)blockIdx.y * 64;
    __shared__ int32_t pos[64];
    __shared__ int32_t grow[64];
    __shared__ float As[32][65];
    __shared__ float Bs[32][64];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    if (tid < 64) {
        const int p = tid < cnt ? L.perm[r0 + tid] : -1;
        pos[tid] = p;
        grow[tid] = p >= 0 ? L.chunk[p] : -1;
    }
    __syncthreads();
    const __nv_bfloat16 *Wb = W + (size_t)b * dg * dl;
    float acc[4][4] = {};
    for (int64_t k0 = 0; k0 < dg; k0 += 32) {
        for (int e = tid; e < 64 * 32; e += 256) {
            const int rr = e >> 5, kk = e & 31;
            const int g = grow[rr];
            As[kk][rr] = g >= 0 ? __bfloat162float(G[(int64_t)g * dg + k0 + kk]) : 0.f;
        }
        for (int e = tid; e < 32 * 64; e += 256) {
            const int kk = e >> 6, cc = e & 63;
            Bs[kk][cc] = __bfloat162float(Wb[(k0 + kk) * dl + n0 + cc]);
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            float a[4], bb[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) { a[q] = As[kk][ty * 4 + q]; bb[q] = Bs[kk][tx * 4 + q]; }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[q][r] = fmaf(a[q], bb[r], acc[q][r]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int p = pos[ty * 4 + q];
        if (p < 0) continue;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t j = n0 + tx * 4 + r;
            S[(int64_t)p * dl + j] = ld_f(H + (int64_t)p * dl + j) + acc[q][r];
        }
    }
}

}  // namespace up
}  // namespace dbc

using namespace dbc;

extern "C" size_t chunk_upsample_workspace(int64_t rows, int64_t N, int nbins) {
    (void)rows; (void)nbins;
    if (N < 0) return 0;
    return up::carve(nullptr, N).bytes;
}

extern "C" dbc_status chunk_upsample(const void *G, int64_t d_g, const void *H, int dtype,
                                     const int64_t *offsets, int64_t T, int64_t N, int64_t d_l,
                                     const int64_t *idx, const int64_t *idx_offsets, int64_t rows,
                                     const void *W_bin, int nbins, int mode, float *S, void *ws,
                                     size_t ws_bytes, int32_t *dev_status, dbc_stream_t stream) {
    if (rows < 0 || T < 0 || N < 0 || d_g <= 0 || d_l <= 0) return DBC_ERR_INVALID_ARG;
    if (nbins < 1 || nbins > up::kMaxBins) return DBC_ERR_INVALID_ARG;
    if (mode < DBC_BIN_IN_CHUNK_OFFSET || mode > DBC_BIN_ABSOLUTE) return DBC_ERR_INVALID_ARG;
    if (dtype != DBC_F32 && dtype != DBC_BF16) return DBC_ERR_UNSUPPORTED;
    if (d_g % 64 || d_l % 64 || d_g > 2048 || d_l > 2048) return DBC_ERR_UNSUPPORTED;
    if (!offsets && N != rows * T) return DBC_ERR_INVALID_ARG;
    if (N > INT32_MAX - 1) return DBC_ERR_UNSUPPORTED;
    if (N == 0 || rows == 0) return DBC_OK;
    if (!G || !H || !idx || !idx_offsets || !W_bin || !S) return DBC_ERR_INVALID_ARG;
    const up::Layout need = up::carve(nullptr, N);
    if (!ws || ws_bytes < need.bytes || (reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)))
        return DBC_ERR_WORKSPACE;
    const up::Layout L = up::carve(ws, N);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaMemsetAsync(L.hist, 0, sizeof(int32_t) * up::kMaxBins, s);
    const int sms = num_sms();
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((N + 255) / 256, (int64_t)sms * 8));
    up::classify_kernel<<<grid, 256, 0, s>>>(offsets, T, N, idx, idx_offsets, rows, nbins, mode, L,
                                             dev_status);
    up::scan_bins_kernel<<<1, 32, 0, s>>>(nbins, L);
    up::scatter_kernel<<<grid, 256, 0, s>>>(N, L);
    dim3 g((unsigned)((N + 63) / 64 + nbins), (unsigned)(d_l / 64));
    if (dtype == DBC_BF16)
        up::bin_gemm_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(G), d_g, static_cast<const __nv_bfloat16 *>(H), d_l,
            static_cast<const __nv_bfloat16 *>(W_bin), nbins, L, S);
    else
        up::bin_gemm_kernel<float><<<g, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(G), d_g, static_cast<const float *>(H), d_l,
            static_cast<const __nv_bfloat16 *>(W_bin), nbins, L, S);
    count_launches(4);
    return launch_status();
}

// ---------------------------------------------------------------------------
// chunk_upsample_noalloc: the same computation as chunk_upsample, for callers
// that cannot hand the library a workspace.  Its scratch (per-position chunk
// and bin, the bin permutation and the bin counters) lives in one file-scope
// device array that every GPU loading this library holds until the process
// exits.  Host code never passes that array's name to a kernel (in host code
// it is only a stand-in for the device symbol); the device address is looked
// up once per device with cudaGetSymbolAddress and cached.
// ---------------------------------------------------------------------------
#include <mutex>

namespace dbc {
namespace up {

constexpr int64_t kNoAllocMaxN = 1 << 20;                 // positions per call
constexpr size_t kNoAllocScratchBytes = 10u << 20;        // 10 MiB
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void *g_noalloc_ptr[kNoAllocMaxDevices];

// Device address of the static scratch on the current device (looked up on
// the first call made with that device current, then cached).
static dbc_status noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DBC_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return DBC_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DBC_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return DBC_OK;
}

}  // namespace up
}  // namespace dbc

extern "C" dbc_status chunk_upsample_noalloc(const void *G, int64_t d_g, const void *H, int dtype,
                                             const int64_t *offsets, int64_t T, int64_t N, int64_t d_l,
                                             const int64_t *idx, const int64_t *idx_offsets, int64_t rows,
                                             const void *W_bin, int nbins, int mode, float *S,
                                             int32_t *dev_status, dbc_stream_t stream) {
    if (rows < 0 || T < 0 || N < 0 || d_g <= 0 || d_l <= 0) return DBC_ERR_INVALID_ARG;
    if (nbins < 1 || nbins > up::kMaxBins) return DBC_ERR_INVALID_ARG;
    if (mode < DBC_BIN_IN_CHUNK_OFFSET || mode > DBC_BIN_ABSOLUTE) return DBC_ERR_INVALID_ARG;
    if (dtype != DBC_F32 && dtype != DBC_BF16) return DBC_ERR_UNSUPPORTED;
    if (d_g % 64 || d_l % 64 || d_g > 2048 || d_l > 2048) return DBC_ERR_UNSUPPORTED;
    if (!offsets && N != rows * T) return DBC_ERR_INVALID_ARG;
    if (N > up::kNoAllocMaxN) return DBC_ERR_WORKSPACE;   // larger than the built-in scratch
    if (N == 0 || rows == 0) return DBC_OK;
    if (!G || !H || !idx || !idx_offsets || !W_bin || !S) return DBC_ERR_INVALID_ARG;
    if (up::carve(nullptr, N).bytes > up::kNoAllocScratchBytes) return DBC_ERR_WORKSPACE;
    void *scratch = nullptr;
    const dbc_status ss = up::noalloc_scratch(&scratch);
    if (ss != DBC_OK) return ss;
    const up::Layout L = up::carve(scratch, N);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The bin counters must start at zero; everything else is written before it is read.
    cudaMemsetAsync(L.hist, 0, sizeof(int32_t) * up::kMaxBins, s);
    const int sms = num_sms();
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((N + 255) / 256, (int64_t)sms * 8));
    up::classify_kernel<<<grid, 256, 0, s>>>(offsets, T, N, idx, idx_offsets, rows, nbins, mode, L,
                                             dev_status);
    up::scan_bins_kernel<<<1, 32, 0, s>>>(nbins, L);
    up::scatter_kernel<<<grid, 256, 0, s>>>(N, L);
    dim3 g((unsigned)((N + 63) / 64 + nbins), (unsigned)(d_l / 64));
    if (dtype == DBC_BF16)
        up::bin_gemm_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(G), d_g, static_cast<const __nv_bfloat16 *>(H), d_l,
            static_cast<const __nv_bfloat16 *>(W_bin), nbins, L, S);
    else
        up::bin_gemm_kernel<float><<<g, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(G), d_g, static_cast<const float *>(H), d_l,
            static_cast<const __nv_bfloat16 *>(W_bin), nbins, L, S);
    count_launches(4);
    return launch_status();
}
