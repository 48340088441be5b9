// chunk_upsample_backward and chunk_gather_backward: the gradients that carry
// a training signal through the upsampling (ByteFlow, paper.rainbus.top
// summary, "Method steps", stage 4; papernotes.org notes, "Key design 4") and
// back through the gather of stage 2.  The Top-K selection passes no gradient.
//
// With dS = dL/dS and s_t = h_t + g_{c(t)} W_{b(t)}:
//   dG_k = sum over t in chunk k of dS_t W_{b(t)}^T
//   dW_b = sum over t in bin b of g_{c(t)}^T dS_t
//   dH   = dS (residual), plus dH_{s_k} += dZ_k through the gather.
//
// Inside a chunk the bin never decreases with t (all three bin rules), so the
// positions sharing one (chunk, bin) pair form a run.  Each run is one
// "product": its rows of dS are summed once (D_p), which turns both gradients
// into grouped GEMMs over bins with one row per product:
//   dG[chunk_p] += D_p W_b^T          (per bin, rows = its products)
//   dW_b        += G[chunk_p]^T D_p   (per bin, contraction over its products)
// Both run on tcgen05 (bf16 operands, fp32 accumulators in TMEM).  D is fp32
// and enters as two bf16 pieces (hi + lo, ~2^-17 relative); G and W are bf16
// and exact.  The epilogues add their tiles into dG / dW with vector atomics
// (a chunk's products sit in different bins, a bin's products in several
// CTAs), so the summation order of those few partial sums is not fixed.
#include "bins.cuh"
#include "common.cuh"
#include "tc.cuh"

namespace dbc {
namespace ub {

constexpr int kMaxBins = 64;
constexpr int kBlk = 256;       // positions per block of the run scan
constexpr int kSplit = 512;     // products per CTA of the weight-gradient GEMM
constexpr int kLong = 64;       // runs longer than this are summed by whole CTAs, kTile positions at a time
constexpr int kTile = 256;

struct Layout {
    int32_t *chunk;       // [N] chunk of each position
    uint8_t *bin;         // [N] bin of each position
    int32_t *blk;         // [nblk + 1] run starts per position block, then their exclusive prefix
    int32_t *t0;          // [N + 1] first position of each product; t0[P] = N
    int32_t *pchunk;      // [N] chunk of each product
    uint8_t *pbin;        // [N] bin of each product
    int32_t *slot;        // [N] product -> slot (slots grouped by bin)
    int32_t *schunk;      // [N] slot -> chunk
    int32_t *hist;        // [kMaxBins] products per bin
    int32_t *cursor;      // [kMaxBins]
    int32_t *bin_start;   // [kMaxBins + 1] first slot of each bin
    int32_t *tile_start;  // [kMaxBins + 1] first 128-slot tile of each bin
    int32_t *split_start; // [kMaxBins + 1] first kSplit-slot split of each bin
    int32_t *nprod;       // [1] number of products P
    int32_t *long_pid;    // [N / (kLong + 1) + 1] products whose run is longer than kLong
    int32_t *nlong;       // [1]
    float *Dlong;         // [N / (kLong + 1) + 1][d_l] fp32 sums of the long runs
    __nv_bfloat16 *Dh;    // [N][d_l] per slot: sum of dS over the product's run, high bf16 piece
    __nv_bfloat16 *Dl;    // [N][d_l] low piece
    size_t bytes;
};

inline Layout carve(void *ws, int64_t N, int64_t d_l) {
    Carver c(ws);
    Layout L;
    const int64_t nblk = (N + kBlk - 1) / kBlk;
    L.chunk = c.take<int32_t>(N + 1);
    L.bin = c.take<uint8_t>(N + 1);
    L.blk = c.take<int32_t>(nblk + 1);
    L.t0 = c.take<int32_t>(N + 1);
    L.pchunk = c.take<int32_t>(N + 1);
    L.pbin = c.take<uint8_t>(N + 1);
    L.slot = c.take<int32_t>(N + 1);
    L.schunk = c.take<int32_t>(N + 1);
    L.hist = c.take<int32_t>(kMaxBins);
    L.cursor = c.take<int32_t>(kMaxBins);
    L.bin_start = c.take<int32_t>(kMaxBins + 1);
    L.tile_start = c.take<int32_t>(kMaxBins + 1);
    L.split_start = c.take<int32_t>(kMaxBins + 1);
    L.nprod = c.take<int32_t>(1);
    const int64_t maxlong = N / (kLong + 1) + 1;
    L.long_pid = c.take<int32_t>(maxlong);
    L.nlong = c.take<int32_t>(1);
    L.Dlong = c.take<float>((size_t)maxlong * d_l);
    L.Dh = c.take<__nv_bfloat16>((size_t)N * d_l);
    L.Dl = c.take<__nv_bfloat16>((size_t)N * d_l);
    L.bytes = c.off;
    return L;
}

__global__ void __launch_bounds__(256) classify_kernel(const int64_t *offsets, int64_t T, int64_t N,
                                                       const int64_t *__restrict__ idx,
                                                       const int64_t *__restrict__ idx_offsets, int64_t rows,
                                                       int nbins, int mode, Layout L, int32_t *st) {
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < N;
         p += (int64_t)gridDim.x * blockDim.x) {
        const PosClass pc = classify_position(p, offsets, T, idx, idx_offsets, rows, nbins, mode, st);
        L.chunk[p] = pc.chunk;
        L.bin[p] = (uint8_t)pc.bin;
    }
}

// A product starts where the (chunk, bin) pair changes; chunks are numbered
// over the whole batch, so a row start is always a product start.
__device__ __forceinline__ bool run_start(const Layout &L, int64_t p, int64_t N) {
    return p < N && (p == 0 || L.chunk[p] != L.chunk[p - 1] || L.bin[p] != L.bin[p - 1]);
}

__global__ void __launch_bounds__(kBlk) run_count_kernel(int64_t N, Layout L) {
    const int64_t p = (int64_t)blockIdx.x * kBlk + threadIdx.x;
    const int c = __syncthreads_count(run_start(L, p, N));
    if (threadIdx.x == 0) L.blk[blockIdx.x] = c;
}

// Exclusive prefix of the per-block run counts (one CTA of 1024 threads).
__global__ void __launch_bounds__(1024) scan_blocks_kernel(int64_t nblk, int64_t N, Layout L) {
    __shared__ int32_t wsum[32];
    __shared__ int32_t total;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t carry = 0;
    for (int64_t base = 0; base < nblk; base += 1024) {
        const int64_t i = base + tid;
        const int32_t v = i < nblk ? L.blk[i] : 0;
        int32_t x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int32_t w = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            wsum[lane] = w;                       // inclusive over warps
            if (lane == 31) total = w;
        }
        __syncthreads();
        const int32_t incl = x + (warp > 0 ? wsum[warp - 1] : 0);
        if (i < nblk) L.blk[i] = carry + incl - v;
        carry += total;
        __syncthreads();
    }
    if (tid == 0) {
        L.blk[nblk] = carry;
        *L.nprod = carry;
        L.t0[carry] = (int32_t)N;
    }
}

__global__ void __launch_bounds__(kBlk) emit_kernel(int64_t N, int nbins, Layout L) {
    __shared__ int32_t wcnt[kBlk / 32];
    __shared__ int32_t h[kMaxBins];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int b = tid; b < nbins; b += kBlk) h[b] = 0;
    const int64_t p = (int64_t)blockIdx.x * kBlk + tid;
    const bool f = run_start(L, p, N);
    const unsigned m = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wcnt[warp] = __popc(m);
    __syncthreads();
    int32_t off = L.blk[blockIdx.x];
    for (int w = 0; w < warp; ++w) off += wcnt[w];
    if (f) {
        const int32_t pid = off + __popc(m & ((1u << lane) - 1u));
        const int b = L.bin[p];
        L.t0[pid] = (int32_t)p;
        L.pchunk[pid] = L.chunk[p];
        L.pbin[pid] = (uint8_t)b;
        atomicAdd(&h[b], 1);
    }
    __syncthreads();
    for (int b = tid; b < nbins; b += kBlk)
        if (h[b]) atomicAdd(&L.hist[b], h[b]);
}

__global__ void scan_bins_kernel(int nbins, Layout L) {
    if (threadIdx.x == 0) {
        int32_t s = 0, t = 0, q = 0;
        for (int b = 0; b < nbins; ++b) {
            L.bin_start[b] = s;
            L.tile_start[b] = t;
            L.split_start[b] = q;
            L.cursor[b] = 0;
            s += L.hist[b];
            t += (L.hist[b] + 127) / 128;
            q += (L.hist[b] + kSplit - 1) / kSplit;
        }
        L.bin_start[nbins] = s;
        L.tile_start[nbins] = t;
        L.split_start[nbins] = q;
        *L.nlong = 0;
    }
}

// Products -> slots grouped by bin (one global atomic per bin and block).
__global__ void __launch_bounds__(256) slot_kernel(int nbins, Layout L) {
    __shared__ int32_t cnt[kMaxBins], base[kMaxBins];
    const int64_t P = *L.nprod;
    for (int64_t p0 = (int64_t)blockIdx.x * blockDim.x; p0 < P; p0 += (int64_t)gridDim.x * blockDim.x) {
        for (int b = threadIdx.x; b < nbins; b += blockDim.x) cnt[b] = 0;
        __syncthreads();
        const int64_t pid = p0 + threadIdx.x;
        int b = -1, local = 0;
        if (pid < P) {
            b = L.pbin[pid];
            local = atomicAdd(&cnt[b], 1);
        }
        __syncthreads();
        for (int q = threadIdx.x; q < nbins; q += blockDim.x)
            base[q] = cnt[q] ? atomicAdd(&L.cursor[q], cnt[q]) : 0;
        __syncthreads();
        if (b >= 0) {
            const int32_t s = L.bin_start[b] + base[b] + local;
            L.slot[pid] = s;
            L.schunk[s] = L.pchunk[pid];
        }
        __syncthreads();
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a)) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b)) << 16);
}

__device__ __forceinline__ void store_pieces(__nv_bfloat16 *Dh, __nv_bfloat16 *Dl, int64_t off, float4 acc) {
    const float hx = __bfloat162float(__float2bfloat16_rn(acc.x));
    const float hy = __bfloat162float(__float2bfloat16_rn(acc.y));
    const float hz = __bfloat162float(__float2bfloat16_rn(acc.z));
    const float hw = __bfloat162float(__float2bfloat16_rn(acc.w));
    *reinterpret_cast<uint2 *>(Dh + off) = make_uint2(pack_bf16x2(hx, hy), pack_bf16x2(hz, hw));
    *reinterpret_cast<uint2 *>(Dl + off) =
        make_uint2(pack_bf16x2(acc.x - hx, acc.y - hy), pack_bf16x2(acc.z - hz, acc.w - hw));
}

__device__ __forceinline__ void add4(float4 &a, const float4 &x) {
    a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
}

// One warp per product of at most kLong positions: D = sum of its dS rows (in
// position order, four rows in flight), stored as hi + lo bf16 pieces at the
// product's slot; optionally dH = dS on the way.  Longer products are queued
// for long_sum_kernel (their fp32 sum row is cleared here).
__global__ void __launch_bounds__(256) sum_kernel(const float4 *__restrict__ dS, int64_t nv4, float4 *dH,
                                                  Layout L) {
    const int lane = threadIdx.x & 31;
    const int64_t P = *L.nprod;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t pid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); pid < P; pid += nw) {
        const int64_t a = L.t0[pid], e = L.t0[pid + 1];
        if (e - a > kLong) {
            int j = 0;
            if (lane == 0) {
                j = atomicAdd(L.nlong, 1);
                L.long_pid[j] = (int32_t)pid;
            }
            j = __shfl_sync(0xffffffffu, j, 0);
            float4 *row = reinterpret_cast<float4 *>(L.Dlong + (size_t)j * nv4 * 4);
            for (int64_t f = lane; f < nv4; f += 32) row[f] = make_float4(0.f, 0.f, 0.f, 0.f);
            continue;
        }
        const int64_t s = L.slot[pid];
        for (int64_t f = lane; f < nv4; f += 32) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            int64_t t = a;
            for (; t + 4 <= e; t += 4) {
                const float4 x0 = dS[t * nv4 + f], x1 = dS[(t + 1) * nv4 + f];
                const float4 x2 = dS[(t + 2) * nv4 + f], x3 = dS[(t + 3) * nv4 + f];
                add4(acc, x0); add4(acc, x1); add4(acc, x2); add4(acc, x3);
                if (dH) {
                    dH[t * nv4 + f] = x0; dH[(t + 1) * nv4 + f] = x1;
                    dH[(t + 2) * nv4 + f] = x2; dH[(t + 3) * nv4 + f] = x3;
                }
            }
            for (; t < e; ++t) {
                const float4 x = dS[t * nv4 + f];
                add4(acc, x);
                if (dH) dH[t * nv4 + f] = x;
            }
            store_pieces(L.Dh, L.Dl, (s * nv4 + f) * 4, acc);
        }
    }
}

// Long products, split into kTile-position tiles dealt round-robin over the
// CTAs: 4 position groups x 64 float4 columns per pass, partial sums combined
// in shared memory and added into the product's fp32 row.
__global__ void __launch_bounds__(256) long_sum_kernel(const float4 *__restrict__ dS, int64_t nv4, float4 *dH,
                                                       Layout L) {
    __shared__ float4 part[4][64];
    const int tid = threadIdx.x, pg = tid >> 6, fl = tid & 63;
    const int nl = *L.nlong;
    const int64_t G = gridDim.x;
    int64_t tile_base = 0;
    for (int j = 0; j < nl; ++j) {
        const int64_t pid = L.long_pid[j];
        const int64_t a = L.t0[pid], e = L.t0[pid + 1];
        const int64_t ntile = (e - a + kTile - 1) / kTile;
        const int64_t i0 = ((int64_t)blockIdx.x - tile_base % G + G) % G;
        for (int64_t i = i0; i < ntile; i += G) {
            const int64_t p0 = a + i * kTile, p1 = p0 + kTile < e ? p0 + kTile : e;
            for (int64_t fb = 0; fb < nv4; fb += 64) {
                const int64_t f = fb + fl;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                if (f < nv4) {
                    int64_t t = p0 + pg;
                    for (; t + 12 < p1; t += 16) {
                        const float4 x0 = dS[t * nv4 + f], x1 = dS[(t + 4) * nv4 + f];
                        const float4 x2 = dS[(t + 8) * nv4 + f], x3 = dS[(t + 12) * nv4 + f];
                        add4(acc, x0); add4(acc, x1); add4(acc, x2); add4(acc, x3);
                        if (dH) {
                            dH[t * nv4 + f] = x0; dH[(t + 4) * nv4 + f] = x1;
                            dH[(t + 8) * nv4 + f] = x2; dH[(t + 12) * nv4 + f] = x3;
                        }
                    }
                    for (; t < p1; t += 4) {
                        const float4 x = dS[t * nv4 + f];
                        add4(acc, x);
                        if (dH) dH[t * nv4 + f] = x;
                    }
                }
                part[pg][fl] = acc;
                __syncthreads();
                if (pg == 0 && f < nv4) {
                    float4 r = part[0][fl];
                    add4(r, part[1][fl]); add4(r, part[2][fl]); add4(r, part[3][fl]);
                    atomicAdd(reinterpret_cast<float4 *>(L.Dlong + (size_t)j * nv4 * 4) + f, r);
                }
                __syncthreads();
            }
        }
        tile_base += ntile;
    }
}

// One warp per long product: its fp32 sum -> hi + lo pieces at its slot.
__global__ void __launch_bounds__(256) long_final_kernel(int64_t nv4, Layout L) {
    const int lane = threadIdx.x & 31;
    const int nl = *L.nlong;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t j = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < nl; j += nw) {
        const int64_t s = L.slot[L.long_pid[j]];
        const float4 *row = reinterpret_cast<const float4 *>(L.Dlong + (size_t)j * nv4 * 4);
        for (int64_t f = lane; f < nv4; f += 32) store_pieces(L.Dh, L.Dl, (s * nv4 + f) * 4, row[f]);
    }
}

// Adds a 128 x nt fp32 tile, staged in shared memory with row stride LDT, into
// rows dst_row(rr) of a row-major fp32 matrix (row length ld), one row per warp
// step with coalesced float4 atomics.
constexpr int LDT = 260;

// ---------------------------------------------------------------- dG GEMM
// One CTA = 128 slots of one bin x up to 256 columns of d_g.  A = D pieces
// (K-major, K = d_l), B = W_b rows (K-major: row g of W_b is contiguous in l).
struct DgTC {
    static constexpr int NS = 3;
    static constexpr uint32_t A_BYTES = 128 * 128;              // 128 rows x 64 K bf16
    static constexpr uint32_t B_BYTES = 256 * 128;              // 256 rows x 64 K bf16
    static constexpr uint32_t STAGE = 2 * A_BYTES + B_BYTES;
    static constexpr size_t SMEM = NS * STAGE + 1024;
};
static_assert(DgTC::NS * DgTC::STAGE >= 128u * LDT * 4u, "epilogue tile must fit in the stages");

__global__ void __launch_bounds__(128, 1) dg_gemm_kernel(const __nv_bfloat16 *__restrict__ W, int64_t dg,
                                                         int64_t dl, int nbins, Layout L, float *dG,
                                                         int64_t total_K, int32_t *st) {
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[DgTC::NS];
    __shared__ uint32_t tmem_base;
    __shared__ int32_t grow[128];
    const int tile = blockIdx.x;
    if (tile >= L.tile_start[nbins]) return;
    int b = 0;
    while (b + 1 < nbins && L.tile_start[b + 1] <= tile) ++b;
    const int r0 = L.bin_start[b] + (tile - L.tile_start[b]) * 128;
    const int cnt = min(128, L.bin_start[b + 1] - r0);
    const int64_t n0 = (int64_t)blockIdx.y * 256;
    const int nt = (int)(dg - n0 < 256 ? dg - n0 : 256);        // multiple of 64
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    {
        int g = tid < cnt ? L.schunk[r0 + tid] : -1;
        if (g >= total_K) {
            flag(st, DBC_ERR_BOUNDS);
            g = -1;
        }
        grow[tid] = g;
    }
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
    if (tid == 0) {
        for (int i = 0; i < DgTC::NS; ++i) tc::mbar_init(&mbar[i], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const __nv_bfloat16 *Wb = W + (size_t)b * dg * dl + (size_t)n0 * dl;
    const int nchunks = (int)(dl / 64);
    auto load = [&](int c, uint32_t sa) {
        for (int e = tid; e < 128 * 8; e += 128) {
            const int r = e >> 3, ch = e & 7;
            const bool in = r < cnt;
            const size_t off = (size_t)(in ? r0 + r : 0) * dl + c * 64 + ch * 8;
            tc::cp_async16(sa + tc::kmajor_off(r, ch * 8), L.Dh + off, in ? 16u : 0u);
            tc::cp_async16(sa + DgTC::A_BYTES + tc::kmajor_off(r, ch * 8), L.Dl + off, in ? 16u : 0u);
        }
        const uint32_t sb = sa + 2 * DgTC::A_BYTES;
        for (int e = tid; e < nt * 8; e += 128) {
            const int r = e >> 3, ch = e & 7;
            tc::cp_async16(sb + tc::kmajor_off(r, ch * 8), Wb + (size_t)r * dl + c * 64 + ch * 8, 16u);
        }
    };
    const uint32_t idesc = tc::idesc_bf16(128, nt, false, false);
    bool ok = true;
    for (int c = 0; c < DgTC::NS - 1; ++c) {
        if (c < nchunks) load(c, base + (uint32_t)c * DgTC::STAGE);
        tc::cp_async_commit();
    }
    for (int c = 0; c < nchunks; ++c) {
        const int cn = c + DgTC::NS - 1;
        if (cn < nchunks) {
            if (cn >= DgTC::NS) ok &= tc::mbar_wait(&mbar[cn % DgTC::NS], (uint32_t)((cn / DgTC::NS) - 1) & 1u, st);
            load(cn, base + (uint32_t)(cn % DgTC::NS) * DgTC::STAGE);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<DgTC::NS - 1>();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t sa = base + (uint32_t)(c % DgTC::NS) * DgTC::STAGE, sb = sa + 2 * DgTC::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = tc::sdesc(sb + kk * 32, 16, 1024);
                tc::mma_bf16(tbase, tc::sdesc(sa + kk * 32, 16, 1024), bd, idesc, (c > 0 || kk > 0) ? 1u : 0u);
                tc::mma_bf16(tbase, tc::sdesc(sa + DgTC::A_BYTES + kk * 32, 16, 1024), bd, idesc, 1u);
            }
            tc::mma_commit(&mbar[c % DgTC::NS]);
        }
        __syncthreads();
    }
    if (nchunks > 0) ok &= tc::mbar_wait(&mbar[(nchunks - 1) % DgTC::NS], (uint32_t)((nchunks - 1) / DgTC::NS) & 1u, st);
    ok = __syncthreads_and(ok) != 0;
    tc::fence_after_sync();
    if (ok) {
        tc::cp_async_wait<0>();
        __syncthreads();
        float *tilep = reinterpret_cast<float *>(smraw + (base - tc::smem_u32(smraw)));
        const int r = warp * 32 + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < nt; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
            float4 *d = reinterpret_cast<float4 *>(tilep + r * LDT + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
        __syncthreads();
        const int nv = nt / 4;
#pragma unroll 1
        for (int rr = warp; rr < cnt; rr += 4) {
            const int g = grow[rr];
            if (g < 0) continue;
            float4 *dst = reinterpret_cast<float4 *>(dG + (size_t)g * dg + n0);
            const float4 *src = reinterpret_cast<const float4 *>(tilep + rr * LDT);
            for (int c4 = lane; c4 < nv; c4 += 32) atomicAdd(dst + c4, src[c4]);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}

// ---------------------------------------------------------------- dW GEMM
// One CTA = one kSplit-slot range of one bin x 128 rows of d_g x up to 256
// columns of d_l.  The contraction runs over the products: A = G rows of the
// products' chunks (MN-major: a row of G is contiguous in g), B = D pieces
// (MN-major: a row of D is contiguous in l).
struct DwTC {
    static constexpr int NS = 2;
    static constexpr uint32_t A_BYTES = 2 * 8192;               // 128 g x 64 products
    static constexpr uint32_t B_BYTES = 4 * 8192;               // 256 l x 64 products, one piece
    static constexpr uint32_t STAGE = A_BYTES + 2 * B_BYTES;
    static constexpr size_t SMEM = NS * STAGE + 1024;
};
static_assert(DwTC::NS * DwTC::STAGE >= 128u * LDT * 4u, "epilogue tile must fit in the stages");

__global__ void __launch_bounds__(128, 1) dw_gemm_kernel(const __nv_bfloat16 *__restrict__ G, int64_t dg,
                                                         int64_t dl, int nbins, Layout L, float *dW,
                                                         int64_t total_K, int32_t *st) {
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[DwTC::NS];
    __shared__ uint32_t tmem_base;
    __shared__ int32_t grow[kSplit];
    const int split = blockIdx.x;
    if (split >= L.split_start[nbins]) return;
    int b = 0;
    while (b + 1 < nbins && L.split_start[b + 1] <= split) ++b;
    const int r0 = L.bin_start[b] + (split - L.split_start[b]) * kSplit;
    const int cnt = min(kSplit, L.bin_start[b + 1] - r0);
    const int64_t m0 = (int64_t)blockIdx.y * 128;
    const int64_t n0 = (int64_t)blockIdx.z * 256;
    const int nt = (int)(dl - n0 < 256 ? dl - n0 : 256);        // multiple of 64
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < kSplit; i += 128) {
        int g = i < cnt ? L.schunk[r0 + i] : -1;
        if (g >= total_K) {
            flag(st, DBC_ERR_BOUNDS);
            g = -1;
        }
        grow[i] = g;
    }
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
    if (tid == 0) {
        for (int i = 0; i < DwTC::NS; ++i) tc::mbar_init(&mbar[i], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const int nchunks = (cnt + 63) / 64;
    const int nb8 = nt / 8;
    auto load = [&](int c, uint32_t sa) {
        for (int e = tid; e < 64 * 16; e += 128) {                 // 64 products x 16 units of 8 g
            const int k = e >> 4, m8 = e & 15;
            const int j = c * 64 + k;
            const int g = j < cnt ? grow[j] : -1;
            const __nv_bfloat16 *src = G + (size_t)(g >= 0 ? g : 0) * dg + m0 + m8 * 8;
            tc::cp_async16(sa + tc::mnmajor_off(m8 * 8, k, 8192), src, g >= 0 ? 16u : 0u);
        }
        const uint32_t sb = sa + DwTC::A_BYTES;
        for (int e = tid; e < 64 * nb8; e += 128) {                // 64 products x nt/8 units of 8 l
            const int k = e / nb8, n8 = e - (e / nb8) * nb8;
            const int j = c * 64 + k;
            const bool in = j < cnt;
            const size_t off = (size_t)(in ? r0 + j : 0) * dl + n0 + n8 * 8;
            const uint32_t o = tc::mnmajor_off(n8 * 8, k, 8192);
            tc::cp_async16(sb + o, L.Dh + off, in ? 16u : 0u);
            tc::cp_async16(sb + DwTC::B_BYTES + o, L.Dl + off, in ? 16u : 0u);
        }
    };
    const uint32_t idesc = tc::idesc_bf16(128, nt, true, true);
    bool ok = true;
    for (int c = 0; c < DwTC::NS - 1; ++c) {
        if (c < nchunks) load(c, base + (uint32_t)c * DwTC::STAGE);
        tc::cp_async_commit();
    }
    for (int c = 0; c < nchunks; ++c) {
        const int cn = c + DwTC::NS - 1;
        if (cn < nchunks) {
            if (cn >= DwTC::NS) ok &= tc::mbar_wait(&mbar[cn % DwTC::NS], (uint32_t)((cn / DwTC::NS) - 1) & 1u, st);
            load(cn, base + (uint32_t)(cn % DwTC::NS) * DwTC::STAGE);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<DwTC::NS - 1>();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t sa = base + (uint32_t)(c % DwTC::NS) * DwTC::STAGE, sb = sa + DwTC::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = tc::sdesc(sa + kk * 2048, 8192, 1024);
                tc::mma_bf16(tbase, ad, tc::sdesc(sb + kk * 2048, 8192, 1024), idesc, (c > 0 || kk > 0) ? 1u : 0u);
                tc::mma_bf16(tbase, ad, tc::sdesc(sb + DwTC::B_BYTES + kk * 2048, 8192, 1024), idesc, 1u);
            }
            tc::mma_commit(&mbar[c % DwTC::NS]);
        }
        __syncthreads();
    }
    if (nchunks > 0) ok &= tc::mbar_wait(&mbar[(nchunks - 1) % DwTC::NS], (uint32_t)((nchunks - 1) / DwTC::NS) & 1u, st);
    ok = __syncthreads_and(ok) != 0;
    tc::fence_after_sync();
    if (ok && nchunks > 0) {
        tc::cp_async_wait<0>();
        __syncthreads();
        float *tilep = reinterpret_cast<float *>(smraw + (base - tc::smem_u32(smraw)));
        const int r = warp * 32 + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < nt; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
            float4 *d = reinterpret_cast<float4 *>(tilep + r * LDT + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
        __syncthreads();
        const int nv = nt / 4;
        float *Wb = dW + (size_t)b * dg * dl;
#pragma unroll 1
        for (int rr = warp; rr < 128; rr += 4) {
            float4 *dst = reinterpret_cast<float4 *>(Wb + (size_t)(m0 + rr) * dl + n0);
            const float4 *src = reinterpret_cast<const float4 *>(tilep + rr * LDT);
            for (int c4 = lane; c4 < nv; c4 += 32) atomicAdd(dst + c4, src[c4]);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}

// ---------------------------------------------------------------- gather adjoint
// One warp per chunk: dH[row start + s_k] (+)= dZ_k.  Boundaries are distinct
// positions, so no two warps touch one row.
__global__ void __launch_bounds__(256) gather_bwd_kernel(const float4 *__restrict__ dZ, int64_t nv4,
                                                         const int64_t *offsets, int64_t T,
                                                         const int64_t *__restrict__ idx,
                                                         const int64_t *__restrict__ idx_offsets, int64_t rows,
                                                         int64_t total, float4 *dH, int accumulate, int32_t *st) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t k = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); k < total; k += warps) {
        const int64_t r = find_row(idx_offsets, rows, k);
        int64_t a, n;
        row_bounds(offsets, r, T, a, n);
        const int64_t t = idx[k];
        if (t < 0 || t >= n) {
            if (lane == 0) flag(st, DBC_ERR_BOUNDS);
            continue;
        }
        float4 *dst = dH + (a + t) * nv4;
        const float4 *src = dZ + k * nv4;
        for (int64_t v = lane; v < nv4; v += 32) {
            float4 x = src[v];
            if (accumulate) {
                const float4 y = dst[v];
                x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
            }
            dst[v] = x;
        }
    }
}

}  // namespace ub
}  // namespace dbc

using namespace dbc;

extern "C" size_t chunk_upsample_backward_workspace(int64_t rows, int64_t N, int nbins, int64_t d_l) {
    (void)rows; (void)nbins;
    if (N < 0 || d_l <= 0) return 0;
    return ub::carve(nullptr, N, d_l).bytes;
}

extern "C" dbc_status chunk_upsample_backward(const float *dS, const void *G, int64_t d_g, const int64_t *offsets,
                                              int64_t T, int64_t N, int64_t d_l, const int64_t *idx,
                                              const int64_t *idx_offsets, int64_t rows, int64_t total_K,
                                              const void *W_bin, int nbins, int mode, float *dG, float *dW,
                                              float *dH, void *ws, size_t ws_bytes, int32_t *dev_status,
                                              dbc_stream_t stream) {
    DBC_NVTX_RANGE("chunk_upsample_backward");
    if (rows < 0 || T < 0 || N < 0 || total_K < 0 || d_g <= 0 || d_l <= 0) return DBC_ERR_INVALID_ARG;
    if (nbins < 1 || nbins > ub::kMaxBins) return DBC_ERR_INVALID_ARG;
    if (mode < DBC_BIN_IN_CHUNK_OFFSET || mode > DBC_BIN_ABSOLUTE) return DBC_ERR_INVALID_ARG;
    if (d_g % 128 || d_l % 64 || d_g > 4096 || d_l > 4096) return DBC_ERR_UNSUPPORTED;
    if (!offsets && N != rows * T) return DBC_ERR_INVALID_ARG;
    if (N > INT32_MAX - 1) return DBC_ERR_UNSUPPORTED;
    if (!dG || !dW) return DBC_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // dG and dW are sums: zero first, also for an empty batch
    cudaMemsetAsync(dW, 0, sizeof(float) * (size_t)nbins * d_g * d_l, s);
    if (total_K > 0) cudaMemsetAsync(dG, 0, sizeof(float) * (size_t)total_K * d_g, s);
    if (N == 0 || rows == 0) return launch_status();
    if (!dS || !G || !idx || !idx_offsets || !W_bin) return DBC_ERR_INVALID_ARG;
    if (!aligned16(dS) || !aligned16(G) || !aligned16(W_bin) || !aligned16(dG) || !aligned16(dW) ||
        (dH && !aligned16(dH)))
        return DBC_ERR_INVALID_ARG;
    const ub::Layout need = ub::carve(nullptr, N, d_l);
    if (!ws || ws_bytes < need.bytes || (reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)))
        return DBC_ERR_WORKSPACE;
    const ub::Layout L = ub::carve(ws, N, d_l);
    cudaMemsetAsync(L.hist, 0, sizeof(int32_t) * ub::kMaxBins, s);
    const int sms = num_sms();
    const int64_t nblk = (N + ub::kBlk - 1) / ub::kBlk;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(nblk, (int64_t)sms * 8));
    ub::classify_kernel<<<grid, 256, 0, s>>>(offsets, T, N, idx, idx_offsets, rows, nbins, mode, L, dev_status);
    ub::run_count_kernel<<<(unsigned)nblk, ub::kBlk, 0, s>>>(N, L);
    ub::scan_blocks_kernel<<<1, 1024, 0, s>>>(nblk, N, L);
    ub::emit_kernel<<<(unsigned)nblk, ub::kBlk, 0, s>>>(N, nbins, L);
    ub::scan_bins_kernel<<<1, 32, 0, s>>>(nbins, L);
    ub::slot_kernel<<<grid, 256, 0, s>>>(nbins, L);
    const int64_t wgrid = std::max<int64_t>(1, std::min<int64_t>((N + 7) / 8, (int64_t)sms * 16));
    ub::sum_kernel<<<(unsigned)wgrid, 256, 0, s>>>(reinterpret_cast<const float4 *>(dS), d_l / 4,
                                                   reinterpret_cast<float4 *>(dH), L);
    ub::long_sum_kernel<<<(unsigned)(2 * sms), 256, 0, s>>>(reinterpret_cast<const float4 *>(dS), d_l / 4,
                                                            reinterpret_cast<float4 *>(dH), L);
    ub::long_final_kernel<<<(unsigned)sms, 256, 0, s>>>(d_l / 4, L);
    cudaFuncSetAttribute(ub::dg_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ub::DgTC::SMEM);
    dim3 gg((unsigned)((N + 127) / 128 + nbins), (unsigned)((d_g + 255) / 256));
    ub::dg_gemm_kernel<<<gg, 128, ub::DgTC::SMEM, s>>>(static_cast<const __nv_bfloat16 *>(W_bin), d_g, d_l, nbins,
                                                      L, dG, total_K, dev_status);
    cudaFuncSetAttribute(ub::dw_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ub::DwTC::SMEM);
    dim3 gw((unsigned)((N + ub::kSplit - 1) / ub::kSplit + nbins), (unsigned)(d_g / 128),
            (unsigned)((d_l + 255) / 256));
    ub::dw_gemm_kernel<<<gw, 128, ub::DwTC::SMEM, s>>>(static_cast<const __nv_bfloat16 *>(G), d_g, d_l, nbins, L,
                                                      dW, total_K, dev_status);
    count_launches(11);
    return launch_status();
}

extern "C" dbc_status chunk_gather_backward(const float *dZ, int64_t d, const int64_t *offsets, int64_t T,
                                            const int64_t *idx, const int64_t *idx_offsets, int64_t rows,
                                            int64_t total_K, float *dH, int accumulate, int32_t *dev_status,
                                            dbc_stream_t stream) {
    DBC_NVTX_RANGE("chunk_gather_backward");
    if (rows < 0 || T < 0 || total_K < 0 || d <= 0) return DBC_ERR_INVALID_ARG;
    if (d % 4) return DBC_ERR_UNSUPPORTED;
    if (total_K == 0 || rows == 0) return DBC_OK;
    if (!dZ || !idx || !idx_offsets || !dH || !aligned16(dZ) || !aligned16(dH)) return DBC_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int sms = num_sms();
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((total_K + 7) / 8, (int64_t)sms * 16));
    ub::gather_bwd_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4 *>(dZ), d / 4, offsets, T, idx,
                                               idx_offsets, rows, total_K, reinterpret_cast<float4 *>(dH),
                                               accumulate, dev_status);
    count_launches(1);
    return launch_status();
}
