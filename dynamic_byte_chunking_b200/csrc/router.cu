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
#include "tc.cuh"

namespace dbc {
namespace rt {

constexpr int kEmaBlk = 64;   // chunks per scan block

struct Layout {
    float *qk;        // [N, 2d]: q in columns [0, d), k in [d, 2d)   (d > 256 only)
    int64_t *count;   // [rows]
    float *ema_a;     // [nblk, d] per-block affine map z_out = a z_in + b
    float *ema_b;     // [nblk, d]
    float *ema_z;     // [nblk, d] value entering each block
    size_t bytes;
};

inline Layout carve(void *ws, int64_t rows, int64_t N, int64_t d) {
    Carver c(ws);
    Layout L;
    L.qk = c.take<float>(d > 256 ? (size_t)N * 2 * d : 0);   // fp32 q|k only for the d > 256 path
    L.count = c.take<int64_t>(rows + 1);
    const int64_t nblk = N / kEmaBlk + 1;
    L.ema_a = c.take<float>((size_t)nblk * d);
    L.ema_b = c.take<float>((size_t)nblk * d);
    L.ema_z = c.take<float>((size_t)nblk * d);
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

// q/k projections on tcgen05 with the cosine epilogue fused.  One CTA = 128
// consecutive positions r0 .. r0+127.  The K-projection reads the rows shifted
// by one (r0-1 .. r0+126), so TMEM lane i holds q_{r0+i} in columns [0, D) and
// k_{r0+i-1} in columns [D, 2D): every thread finishes its own position.
template <int D>
struct RouterTC {
    static constexpr int NS = 2;
    static constexpr uint32_t A_BYTES = 128 * 128;
    static constexpr uint32_t W_BYTES = D * 128;              // 64 K-rows x D columns, MN-major
    static constexpr uint32_t STAGE = 2 * A_BYTES + 2 * W_BYTES;
    static constexpr size_t SMEM = NS * STAGE + 1024;
    static constexpr int TCOLS = 2 * D < 32 ? 32 : 2 * D;
};

template <int D>
__global__ void __launch_bounds__(128, 1) router_tc_kernel(const __nv_bfloat16 *__restrict__ H,
                                                           const int64_t *offsets, int64_t rows, int64_t T,
                                                           int64_t N, const __nv_bfloat16 *__restrict__ Wq,
                                                           const __nv_bfloat16 *__restrict__ Wk, float threshold,
                                                           float *p, uint8_t *bnd, int32_t *st) {
    using C = RouterTC<D>;
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[C::NS];
    __shared__ uint32_t tmem_base;
    const int64_t r0 = (int64_t)blockIdx.x * 128;
    if (r0 >= N) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    if (warp == 0) tc::tmem_alloc(&tmem_base, C::TCOLS);
    if (tid == 0) {
        for (int i = 0; i < C::NS; ++i) tc::mbar_init(&mbar[i], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    constexpr int NCH = D / 64, NB8 = D / 8;
    auto load = [&](int c, uint32_t sa) {
        for (int e = tid; e < 2 * 128 * 8; e += 128) {
            const int which = e >> 10, r = (e >> 3) & 127, ch = e & 7;
            const int64_t t = r0 + r - which;                  // which = 1: shifted rows for k
            const bool in = t >= 0 && t < N;
            tc::cp_async16(sa + which * C::A_BYTES + tc::kmajor_off(r, ch * 8),
                           H + (in ? t : 0) * D + c * 64 + ch * 8, in ? 16u : 0u);
        }
        const uint32_t sw = sa + 2 * C::A_BYTES;
        for (int e = tid; e < 2 * 64 * NB8; e += 128) {
            const int which = e / (64 * NB8), rem = e - which * (64 * NB8);
            const int k = rem / NB8, n8 = rem - (rem / NB8) * NB8;
            const __nv_bfloat16 *W = which ? Wk : Wq;
            tc::cp_async16(sw + which * C::W_BYTES + tc::mnmajor_off(n8 * 8, k, 8192),
                           W + (size_t)(c * 64 + k) * D + n8 * 8, 16u);
        }
    };
    constexpr uint32_t idesc = tc::idesc_bf16(128, D, false, true);
    bool ok = true;
    for (int c = 0; c < C::NS - 1; ++c) {
        if (c < NCH) load(c, base + (uint32_t)c * C::STAGE);
        tc::cp_async_commit();
    }
    for (int c = 0; c < NCH; ++c) {
        const int cn = c + C::NS - 1;
        if (cn < NCH) {
            if (cn >= C::NS) ok &= tc::mbar_wait(&mbar[cn % C::NS], (uint32_t)((cn / C::NS) - 1) & 1u, st);
            load(cn, base + (uint32_t)(cn % C::NS) * C::STAGE);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<C::NS - 1>();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t sa = base + (uint32_t)(c % C::NS) * C::STAGE, sw = sa + 2 * C::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
                tc::mma_bf16(tbase, tc::sdesc(sa + kk * 32, 16, 1024), tc::sdesc(sw + kk * 2048, 8192, 1024), idesc,
                             acc);
                tc::mma_bf16(tbase + D, tc::sdesc(sa + C::A_BYTES + kk * 32, 16, 1024),
                             tc::sdesc(sw + C::W_BYTES + kk * 2048, 8192, 1024), idesc, acc);
            }
            tc::mma_commit(&mbar[c % C::NS]);
        }
        __syncthreads();
    }
    ok &= tc::mbar_wait(&mbar[(NCH - 1) % C::NS], (uint32_t)((NCH - 1) / C::NS) & 1u, st);
    ok = __syncthreads_and(ok) != 0;
    tc::fence_after_sync();
    if (ok) {
        const int64_t t = r0 + warp * 32 + lane;
        float dot = 0.f, nq = 0.f, nk = 0.f;
        const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
            float q[16], k[16];
            tc::tmem_ld16(tl + (uint32_t)c0, q);
            tc::tmem_ld16(tl + (uint32_t)(D + c0), k);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                dot = fmaf(q[i], k[i], dot);
                nq = fmaf(q[i], q[i], nq);
                nk = fmaf(k[i], k[i], nk);
            }
        }
        if (t < N) {
            bool first;
            if (offsets) {
                const int64_t r = find_row(offsets, rows, t);
                first = offsets[r] == t;
            } else {
                first = (t % T) == 0;
            }
            float pv = 1.f;
            if (!first) {
                const float cs = (nq > 0.f && nk > 0.f) ? dot / (sqrtf(nq) * sqrtf(nk)) : 0.f;
                pv = 0.5f * (1.f - cs);
            }
            if (!isfinite(pv)) flag(st, DBC_ERR_NONFINITE);
            p[t] = pv;
            bnd[t] = pv >= threshold ? 1 : 0;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, C::TCOLS);
}

template <int D>
void launch_router_tc(const __nv_bfloat16 *H, const int64_t *offsets, int64_t rows, int64_t T, int64_t N,
                      const __nv_bfloat16 *Wq, const __nv_bfloat16 *Wk, float threshold, float *p, uint8_t *b,
                      int32_t *st, cudaStream_t s) {
    cudaFuncSetAttribute(router_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RouterTC<D>::SMEM);
    router_tc_kernel<D><<<(unsigned)((N + 127) / 128), 128, RouterTC<D>::SMEM, s>>>(H, offsets, rows, T, N, Wq, Wk,
                                                                                   threshold, p, b, st);
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

// EMA over the rows-stacked chunk list as one sequence: p = 1 at every row's
// first position, so the recurrence restarts there by itself.  Three passes:
// per 64-chunk block the affine map z_out = a z_in + b (parallel over blocks
// and features), the chain of block maps, then the recomputation inside blocks.
__device__ __forceinline__ void chunk_source(const int64_t *offsets, int64_t rows, int64_t T, const int64_t *co,
                                             const int64_t *chunk_idx, int64_t j, int64_t &pos) {
    const int64_t r = find_row(co, rows, j);
    int64_t a, n;
    row_bounds(offsets, r, T, a, n);
    pos = a + chunk_idx[j];
}

template <class IN, bool FINAL>
__global__ void __launch_bounds__(256) ema_block_kernel(const IN *__restrict__ H, const int64_t *offsets,
                                                        int64_t rows, int64_t T, int64_t d, const float *p,
                                                        const int64_t *co, const int64_t *chunk_idx, Layout L,
                                                        float *z) {
    __shared__ int64_t spos[kEmaBlk];
    __shared__ float sP[kEmaBlk];
    const int64_t total = co[rows];
    const int64_t j0 = (int64_t)blockIdx.x * kEmaBlk;
    if (j0 >= total) return;
    const int cnt = (int)(total - j0 < kEmaBlk ? total - j0 : kEmaBlk);
    if (threadIdx.x < cnt) {
        int64_t pos;
        chunk_source(offsets, rows, T, co, chunk_idx, j0 + threadIdx.x, pos);
        spos[threadIdx.x] = pos;
        sP[threadIdx.x] = p[pos];
    }
    __syncthreads();
    for (int64_t f = threadIdx.x; f < d; f += blockDim.x) {
        if (!FINAL) {
            float a = 1.f, b = 0.f;
            for (int j = 0; j < cnt; ++j) {
                const float P = sP[j];
                a = (1.f - P) * a;
                b = P * ld_f(H + spos[j] * d + f) + (1.f - P) * b;
            }
            L.ema_a[blockIdx.x * d + f] = a;
            L.ema_b[blockIdx.x * d + f] = b;
        } else {
            float acc = L.ema_z[blockIdx.x * d + f];
            for (int j = 0; j < cnt; ++j) {
                const float P = sP[j];
                acc = P * ld_f(H + spos[j] * d + f) + (1.f - P) * acc;
                z[(j0 + j) * d + f] = acc;
            }
        }
    }
}

__global__ void __launch_bounds__(256) ema_chain_kernel(int64_t rows, int64_t d, const int64_t *co, Layout L) {
    const int64_t total = co[rows];
    const int64_t nblk = (total + kEmaBlk - 1) / kEmaBlk;
    const int64_t f = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (f >= d) return;
    float zc = 0.f;
    int64_t b = 0;
    for (; b + 4 <= nblk; b += 4) {
        float a[4], bb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) { a[q] = L.ema_a[(b + q) * d + f]; bb[q] = L.ema_b[(b + q) * d + f]; }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            L.ema_z[(b + q) * d + f] = zc;
            zc = a[q] * zc + bb[q];
        }
    }
    for (; b < nblk; ++b) {
        L.ema_z[b * d + f] = zc;
        zc = L.ema_a[b * d + f] * zc + L.ema_b[b * d + f];
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
    DBC_NVTX_RANGE("hnet_route");
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
    const __nv_bfloat16 *Wqb = static_cast<const __nv_bfloat16 *>(Wq), *Wkb = static_cast<const __nv_bfloat16 *>(Wk);
    if (d <= 256) {
        switch (d) {
            case 64: rt::launch_router_tc<64>(Hb, offsets, rows, T, N, Wqb, Wkb, threshold, p, boundary, dev_status, s); break;
            case 128: rt::launch_router_tc<128>(Hb, offsets, rows, T, N, Wqb, Wkb, threshold, p, boundary, dev_status, s); break;
            default: rt::launch_router_tc<256>(Hb, offsets, rows, T, N, Wqb, Wkb, threshold, p, boundary, dev_status, s);
        }
    } else {
        dim3 g((unsigned)((N + 63) / 64), (unsigned)(d / 64));
        gemm_bf16_simt<RowIdentity><<<g, 256, 0, s>>>(Hb, d, Wqb, d, L.qk, 2 * d, nullptr, 0, N, d, d, RowIdentity{});
        gemm_bf16_simt<RowIdentity><<<g, 256, 0, s>>>(Hb, d, Wkb, d, L.qk + d, 2 * d, nullptr, 0, N, d, d,
                                                      RowIdentity{});
        const int sms = num_sms();
        const int pg = (int)std::max<int64_t>(1, std::min<int64_t>((N + 7) / 8, (int64_t)sms * 32));
        rt::prob_kernel<<<pg, 256, 0, s>>>(L.qk, offsets, rows, T, N, d, threshold, p, boundary, dev_status);
    }
    const int rg = (int)std::min<int64_t>(rows, 65535);
    rt::count_kernel<<<rg, 1024, 0, s>>>(boundary, offsets, rows, T, L.count);
    rt::offsets_kernel<<<1, 1024, 0, s>>>(L.count, rows, chunk_offsets);
    rt::compact_kernel<<<rg, 1024, 0, s>>>(boundary, offsets, rows, T, chunk_offsets, chunk_idx);
    count_launches((d <= 256 ? 4 : 6) + (do_ema ? 3 : 0));
    if (do_ema) {
        const unsigned nblk = (unsigned)(N / rt::kEmaBlk + 1);
        rt::ema_block_kernel<__nv_bfloat16, false><<<nblk, 256, 0, s>>>(Hb, offsets, rows, T, d, p, chunk_offsets,
                                                                        chunk_idx, L, z_smooth);
        rt::ema_chain_kernel<<<(unsigned)((d + 255) / 256), 256, 0, s>>>(rows, d, chunk_offsets, L);
        rt::ema_block_kernel<__nv_bfloat16, true><<<nblk, 256, 0, s>>>(Hb, offsets, rows, T, d, p, chunk_offsets,
                                                                       chunk_idx, L, z_smooth);
    }
    return launch_status();
}
