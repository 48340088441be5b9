// chunk_upsample: multi-linear upsampling with residual.
//
// ByteFlow (paper.rainbus.top summary, "Method steps", stage 4; papernotes.org
// notes, "Key design 4"): each position t belongs to chunk c(t), the last
// boundary s_c <= t; it falls into one of B bins with its own matrix W_b, and
// S_t = h_t + g_{c(t)} W_{b(t)}.
//
// Positions are classified (chunk, bin), counted per bin and permuted so that
// each bin's positions are contiguous; the product is then a grouped GEMM over
// bins on tcgen05 whose A rows are gathered chunk vectors and whose output rows
// are scattered back to their positions with the residual added.
#include "bins.cuh"
#include "common.cuh"
#include "tc.cuh"
#include "tma_host.cuh"

namespace dbc {
namespace up {

constexpr int kMaxBins = 64;

struct Layout {
    int32_t *chunk;      // [N] global chunk row of each position
    uint8_t *bin;        // [N]
    int32_t *perm;       // [N] positions grouped by bin
    int32_t *hist;       // [kMaxBins]
    int32_t *cursor;     // [kMaxBins]
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
    // a warp classifies 32 consecutive positions together; one shared atomic per distinct bin
    const int lane = threadIdx.x & 31;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < N; base += (int64_t)gridDim.x * blockDim.x) {
        const int64_t p0 = base + (threadIdx.x & ~31);
        if (p0 >= N) continue;                                   // warp-uniform
        const PosClass pc = classify_warp(p0, N, offsets, T, idx, idx_offsets, rows, nbins, mode, st);
        const int64_t p = p0 + lane;
        const bool live = p < N;
        if (live) {
            L.chunk[p] = pc.chunk;
            L.bin[p] = (uint8_t)pc.bin;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, live ? pc.bin : -1);
        if (live && lane == __ffs(peers) - 1) atomicAdd(&h[pc.bin], __popc(peers));
    }
    __syncthreads();
    for (int b = threadIdx.x; b < nbins; b += blockDim.x)
        if (h[b]) atomicAdd(&L.hist[b], h[b]);
}

// Bin tables from the bin counts, computed by one warp of each CTA that needs them (at most 64
// bins): bs[b] = first permutation slot of bin b, ts[b] = first 128-slot tile of bin b, each with
// the total at index nbins.
__device__ __forceinline__ void bin_tables(const int32_t *__restrict__ hist, int nbins, int32_t *bs, int32_t *ts) {
    const int lane = threadIdx.x & 31;
    const int b0 = 2 * lane, b1 = 2 * lane + 1;
    const int32_t h0 = b0 < nbins ? hist[b0] : 0, h1 = b1 < nbins ? hist[b1] : 0;
    const int32_t t0 = (h0 + 127) / 128, t1 = (h1 + 127) / 128;
    int32_t hs = h0 + h1, tsum = t0 + t1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, hs, o), z = __shfl_up_sync(0xffffffffu, tsum, o);
        if (lane >= o) { hs += y; tsum += z; }
    }
    const int32_t he = hs - h0 - h1, te = tsum - t0 - t1;     // exclusive
    if (b0 < nbins) { bs[b0] = he; ts[b0] = te; }
    if (b1 < nbins) { bs[b1] = he + h0; ts[b1] = te + t0; }
    if (lane == 31) { bs[nbins] = hs; ts[nbins] = tsum; }      // the totals (bins past nbins count 0)
}

// Positions -> their bin's slice of the permutation.  Slots are reserved per
// block (one global atomic per bin and block), then handed out in shared memory.
__global__ void __launch_bounds__(256) scatter_kernel(int64_t N, int nbins, Layout L) {
    __shared__ int32_t cnt[kMaxBins], base[kMaxBins];
    __shared__ int32_t s_bs[kMaxBins + 1], s_ts[kMaxBins + 1];
    if (threadIdx.x < 32) bin_tables(L.hist, nbins, s_bs, s_ts);
    __syncthreads();
    for (int64_t p0 = (int64_t)blockIdx.x * blockDim.x; p0 < N; p0 += (int64_t)gridDim.x * blockDim.x) {
        for (int b = threadIdx.x; b < nbins; b += blockDim.x) cnt[b] = 0;
        __syncthreads();
        const int64_t p = p0 + threadIdx.x;
        int b = -1, slot = 0;
        if (p < N) {
            b = L.bin[p];
            slot = atomicAdd(&cnt[b], 1);
        }
        __syncthreads();
        for (int q = threadIdx.x; q < nbins; q += blockDim.x)
            base[q] = cnt[q] ? atomicAdd(&L.cursor[q], cnt[q]) : 0;
        __syncthreads();
        if (b >= 0) L.perm[s_bs[b] + base[b] + slot] = (int32_t)p;
        __syncthreads();
    }
}

// Grouped GEMM on tcgen05: one CTA = 128 positions of one bin x up to 256
// output columns.  A = the positions' chunk vectors g_c (gathered rows,
// K-major, cp.async by all threads), B = W_b (row-major [d_g][d_l], read
// MN-major, TMA tile loads issued by one thread: tensor map over this GPU's own
// memory, no multicast), fp32 accumulators in TMEM; the epilogue adds h_t and
// scatters the rows back to their positions.  Two stages of 48 KB keep the CTA
// small enough for two per SM (with bf16 h), so one CTA's epilogue stores run
// under the other's loads and MMAs.  The tile's residual values are loaded into
// registers early: the first column half's as soon as the positions are known,
// the second half's right after the first K chunk's operand loads (so those go
// out first).  Each CTA lives for one tile, so the DRAM reads it keeps in flight
// are what bounds the kernel (issuing the second half's loads only during the
// first half's stores cost a quarter of the time on the ragged batch).
struct BinTC {
    static constexpr int NS = 2;
    static constexpr uint32_t A_BYTES = 128 * 128;             // 128 rows x 64 K, K-major
    static constexpr uint32_t B_BYTES = 4 * 64 * 128;          // up to 256 columns x 64 K, MN-major
    static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
    static constexpr int LDT = 132;                            // epilogue tile: [128][LDT] fp32, one column half
    static_assert(128u * LDT * 4u <= NS * STAGE, "the epilogue tile reuses the stages");
    static constexpr size_t SMEM = NS * STAGE + 1024;
};

// Four consecutive residual values of a row (8 bytes of bf16 or 16 of fp32).
template <class IN> struct Res4;
template <> struct Res4<__nv_bfloat16> {
    using V = uint2;
    static __device__ __forceinline__ V load(const __nv_bfloat16 *p) { return __ldg(reinterpret_cast<const uint2 *>(p)); }
    static __device__ __forceinline__ void unpack(const V &v, float (&h)[4]) {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&v.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&v.y);
        h[0] = __low2float(a); h[1] = __high2float(a); h[2] = __low2float(b); h[3] = __high2float(b);
    }
};
template <> struct Res4<float> {
    using V = float4;
    static __device__ __forceinline__ V load(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
    static __device__ __forceinline__ void unpack(const V &v, float (&h)[4]) { h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w; }
};

template <class IN>
__global__ void __launch_bounds__(256, sizeof(IN) == 2 ? 2 : 1)
    bin_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __nv_bfloat16 *__restrict__ G, int64_t dg,
                       const IN *__restrict__ H, int64_t dl, int nbins, Layout L, float *__restrict__ S, int64_t N,
                       int32_t *st) {
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[BinTC::NS], wbar[BinTC::NS];      // stage consumed by the MMAs / W_b bytes landed
    __shared__ uint32_t tmem_base;
    __shared__ int32_t pos[128], grow[128];
    __shared__ int32_t s_bs[kMaxBins + 1], s_ts[kMaxBins + 1];
    if (threadIdx.x < 32) bin_tables(L.hist, nbins, s_bs, s_ts);
    __syncthreads();
    const int tile = blockIdx.x;
    if (tile >= s_ts[nbins]) return;
    int b = 0;
    while (b + 1 < nbins && s_ts[b + 1] <= tile) ++b;
    const int r0 = s_bs[b] + (tile - s_ts[b]) * 128;
    const int cnt = min(128, s_bs[b + 1] - r0);
    const int64_t n0 = (int64_t)blockIdx.y * 256;
    const int nt = (int)(dl - n0 < 256 ? dl - n0 : 256);      // multiple of 64
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < 128) pos[tid] = tid < cnt ? L.perm[r0 + tid] : -1;
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
    if (tid == 0) {
        for (int i = 0; i < BinTC::NS; ++i) {
            tc::mbar_init(&mbar[i], 1);
            tc::mbar_init(&wbar[i], 1);
        }
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmW);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    // Residual of row (warp + 8 i), columns half * 128 + lane * 4 .. +3 (zeros for empty rows and
    // columns past the tile): the first half's loads are issued here, before the chunk rows are
    // looked up, the second half's after the first operand loads; they stay in flight through the
    // MMAs
    using R4 = Res4<IN>;
    auto hload = [&](int half, int i) {
        typename R4::V v{};
        const int p = pos[warp + 8 * i];
        const int col = half * 128 + lane * 4;
        if (p >= 0 && p < N && col < nt) v = R4::load(H + (size_t)p * dl + n0 + col);
        return v;
    };
    typename R4::V hr[2][16];
#pragma unroll
    for (int i = 0; i < 16; ++i) hr[0][i] = hload(0, i);
    if (tid < 128) {
        const int p = pos[tid];
        grow[tid] = p >= 0 && p < N ? L.chunk[p] : -1;
    }
    __syncthreads();
    const int nchunks = (int)(dg / 64);
    auto load = [&](int c, uint32_t sa) {
        const uint32_t sb = sa + BinTC::A_BYTES;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + 256 * i;
            const int r = e >> 3, ch = e & 7;
            const int g = grow[r];
            const __nv_bfloat16 *src = G + (size_t)(g >= 0 ? g : 0) * dg + c * 64 + ch * 8;
            tc::cp_async16(sa + tc::kmajor_off(r, ch * 8), src, g >= 0 ? 16u : 0u);
        }
        if (tid == 0) {
            // W_b rows c*64 .. +63, columns n0 .. n0 + nt: nt / 64 boxes of 64 x 64 (8 KB each)
            uint64_t *bar = &wbar[c % BinTC::NS];
            tc::mbar_arrive_expect_tx(bar, (uint32_t)(nt / 64) * 8192u);
            for (int nq = 0; nq < nt / 64; ++nq)
                tc::tma_load_2d(sb + (uint32_t)nq * 8192u, &tmW, bar, (int)(n0 + nq * 64), b * (int)dg + c * 64);
        }
    };
    const uint32_t idesc = tc::idesc_bf16(128, nt, false, true);
    bool ok = true;
    for (int c = 0; c < BinTC::NS - 1; ++c) {
        if (c < nchunks) load(c, base + (uint32_t)c * BinTC::STAGE);
        tc::cp_async_commit();
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) hr[1][i] = hload(1, i);
    for (int c = 0; c < nchunks; ++c) {
        const int cn = c + BinTC::NS - 1;
        if (cn < nchunks) {
            if (cn >= BinTC::NS) ok &= tc::mbar_wait(&mbar[cn % BinTC::NS], (uint32_t)((cn / BinTC::NS) - 1) & 1u, st);
            load(cn, base + (uint32_t)(cn % BinTC::NS) * BinTC::STAGE);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<BinTC::NS - 1>();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            ok &= tc::mbar_wait(&wbar[c % BinTC::NS], (uint32_t)(c / BinTC::NS) & 1u, st);
            tc::fence_after_sync();
            const uint32_t sa = base + (uint32_t)(c % BinTC::NS) * BinTC::STAGE, sb = sa + BinTC::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tbase, tc::sdesc(sa + kk * 32, 16, 1024), tc::sdesc(sb + kk * 2048, 8192, 1024), idesc,
                             (c > 0 || kk > 0) ? 1u : 0u);
            tc::mma_commit(&mbar[c % BinTC::NS]);
        }
        __syncthreads();
    }
    if (nchunks > 0) ok &= tc::mbar_wait(&mbar[(nchunks - 1) % BinTC::NS], (uint32_t)((nchunks - 1) / BinTC::NS) & 1u, st);
    ok = __syncthreads_and(ok) != 0;
    tc::fence_after_sync();
    if (ok) {
        tc::cp_async_wait<0>();
        __syncthreads();
        float *tilep = reinterpret_cast<float *>(smraw + (base - tc::smem_u32(smraw)));
        // per column half: TMEM -> shared tile [128][LDT] (warps w and w + 4 read the same 32 TMEM
        // lanes, each half of the columns), then one coalesced row at a time with the residual added
        const int lg = warp & 3;
        const int r = lg * 32 + lane;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            if (half * 128 >= nt) break;
            const int w = min(128, nt - half * 128);             // 64 or 128 columns
            const int cw = w / 2, cs = (warp >> 2) * cw;
#pragma unroll 1
            for (int c0 = 0; c0 < cw; c0 += 16) {
                float v[16];
                tc::tmem_ld16(tbase + ((uint32_t)(lg * 32) << 16) + (uint32_t)(half * 128 + cs + c0), v);
                float4 *d = reinterpret_cast<float4 *>(tilep + r * BinTC::LDT + cs + c0);
#pragma unroll
                for (int q = 0; q < 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int rr = warp + 8 * i;
                const int p = pos[rr];
                if (p >= 0 && dcheck(p < N, st) && lane * 4 < w) {
                    const float4 a = *reinterpret_cast<const float4 *>(tilep + rr * BinTC::LDT + lane * 4);
                    float h[4];
                    R4::unpack(hr[half][i], h);
                    *reinterpret_cast<float4 *>(S + (size_t)p * dl + n0 + half * 128 + lane * 4) =
                        make_float4(a.x + h[0], a.y + h[1], a.z + h[2], a.w + h[3]);
                }
            }
            __syncthreads();                                     // the tile is rewritten by the next half
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}

// Launch sequence shared by the workspace and the allocation-free entry points.
inline dbc_status launch(const void *G, int64_t d_g, const void *H, int dtype, const int64_t *offsets, int64_t T,
                         int64_t N, int64_t d_l, const int64_t *idx, const int64_t *idx_offsets, int64_t rows,
                         const void *W_bin, int nbins, int mode, float *S, const Layout &L, int32_t *dev_status,
                         cudaStream_t s) {
    // W_bin as one [nbins * d_g][d_l] bf16 matrix read in 64 x 64 boxes (checked before any launch)
    if (reinterpret_cast<uintptr_t>(W_bin) & 15) return DBC_ERR_INVALID_ARG;
    CUtensorMap tmW;
    if (!tma::encode_bf16_rows(&tmW, W_bin, (uint64_t)nbins * (uint64_t)d_g, (uint64_t)d_l, 64)) return DBC_ERR_CUDA;
    // the bin counts and the scatter cursors start at zero (adjacent in the workspace)
    cudaMemsetAsync(L.hist, 0, (size_t)(reinterpret_cast<char *>(L.cursor + kMaxBins) - reinterpret_cast<char *>(L.hist)),
                    s);
    const int sms = num_sms();
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((N + 255) / 256, (int64_t)sms * 8));
    classify_kernel<<<grid, 256, 0, s>>>(offsets, T, N, idx, idx_offsets, rows, nbins, mode, L, dev_status);
    scatter_kernel<<<grid, 256, 0, s>>>(N, nbins, L);
    dim3 g((unsigned)((N + 127) / 128 + nbins), (unsigned)((d_l + 255) / 256));
    if (dtype == DBC_BF16) {
        cudaFuncSetAttribute(bin_gemm_tc_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)BinTC::SMEM);
        // two CTAs per SM need the whole shared-memory carveout
        cudaFuncSetAttribute(bin_gemm_tc_kernel<__nv_bfloat16>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        bin_gemm_tc_kernel<__nv_bfloat16><<<g, 256, BinTC::SMEM, s>>>(
            tmW, static_cast<const __nv_bfloat16 *>(G), d_g, static_cast<const __nv_bfloat16 *>(H), d_l, nbins, L,
            S, N, dev_status);
    } else {
        cudaFuncSetAttribute(bin_gemm_tc_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)BinTC::SMEM);
        bin_gemm_tc_kernel<float><<<g, 256, BinTC::SMEM, s>>>(
            tmW, static_cast<const __nv_bfloat16 *>(G), d_g, static_cast<const float *>(H), d_l, nbins, L, S, N,
            dev_status);
    }
    count_launches(3);
    return launch_status();
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
    DBC_NVTX_RANGE("chunk_upsample");
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
    return up::launch(G, d_g, H, dtype, offsets, T, N, d_l, idx, idx_offsets, rows, W_bin, nbins, mode, S, L,
                      dev_status, reinterpret_cast<cudaStream_t>(stream));
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
    DBC_NVTX_RANGE("chunk_upsample_noalloc");
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
    // launch() clears the bin counters, the only scratch that must start at zero.
    return up::launch(G, d_g, H, dtype, offsets, T, N, d_l, idx, idx_offsets, rows, W_bin, nbins, mode, S, L,
                      dev_status, reinterpret_cast<cudaStream_t>(stream));
}
