// Coding-rate segments on tensor cores (bf16 features, d in {128, 256, 512}).
// Included by coding_rate.cu, which holds the segment table, the tcgen05
// Gram and the float64 first-segment kernel this path shares.
//
// d in {128, 512} (register-panel path), per segment s (rows X_s, start
// state M_s = I + P_s):
//   factor: panel Cholesky of [P_s ; I] with the identity implicit; the
//           appended block becomes B = L_s^{-T} (L_s L_s^T = M_s);
//   ainv:   A_s = B B^T = M_s^{-1}, stored as three bf16 pieces (hi, mid, lo)
//           whose sum carries the fp32 value;
//   vgemm:  V = X_s A_s on tcgen05 (X exact in bf16, three passes over the
//           pieces, fp32 accumulation in TMEM); V stored as three pieces;
//   kgemm:  G'_s = c X_s V^T on tcgen05 (three passes), lower 128-blocks;
//   inseg:  panel Cholesky of I + G'_s with the identity implicit; the
//           excess e_t of each diagonal gives dR_t = log1p(e_t) / 2.
// A row's first segment takes the same path with P = 0 (so A = I).
// G'_s = c X_s M_s^{-1} X_s^T is the in-segment Gram in the frame whitened
// by the segment's start state, so its Cholesky diagonal is the per-position
// Schur complement 1 + c h_t^T M_{t-1}^{-1} h_t (matrix determinant lemma).
// d = 256 (bf16) takes the TMEM path at the end of this file instead: a fused
// TMA-fed Gram + float64 prefix kernel gives every segment's start state, the
// factor kernel keeps B = L_s^{-T} only, and the in-segment kernel forms
// Y = sqrt(c) X_s B on tcgen05 itself and factors I + Y Y^T.
#pragma once

#include "panel_chol.cuh"
#include "tc.cuh"

namespace dbc {
namespace cr {

struct Layout2 {
    Segs segs;
    float *aug2;            // per segment: [2D][D] = [P_s ; I] -> [. ; L^{-T}]
    __nv_bfloat16 *A3;      // per segment: [3][D][D]
    __nv_bfloat16 *V3;      // [3][N][D]
    float *gp;              // per segment at start*kSegMax: len x ldg(len)
    size_t bytes;
};

__host__ __device__ inline int ldg_of(int len) { return (len + 3) & ~3; }

inline Layout2 carve2(void *ws, int64_t rows, int64_t N, int64_t d) {
    Carver c(ws);
    const int64_t ns = nseg_upper(rows, N);
    Layout2 L;
    L.segs.start = c.take<int64_t>(ns);
    L.segs.len = c.take<int32_t>(ns);
    L.segs.row = c.take<int32_t>(ns);
    L.segs.k = c.take<int32_t>(ns);
    L.segs.row_seg0 = c.take<int32_t>(rows + 1);
    L.segs.nseg = c.take<int32_t>(1);
    L.aug2 = c.take<float>((size_t)ns * 2 * d * d);
    L.A3 = c.take<__nv_bfloat16>((size_t)ns * 3 * d * d);
    L.V3 = c.take<__nv_bfloat16>((size_t)3 * N * d + 8);
    L.gp = c.take<float>((size_t)N * kSegMax + 4);
    L.bytes = c.off;
    return L;
}

// ---------------------------------------------------------------- prefix
// In place over a row's segments: Gram -> P_s = c sum_{s'<s} G_s' (float64
// running sum, fp32 store).
// Number of float4 entries of a d x d matrix left of the end of each row's 32-column block.
__host__ __device__ __forceinline__ int64_t lower32_count(int64_t d) {
    const int64_t nb = d / 32;
    return 128 * nb * (nb + 1);
}

__global__ void __launch_bounds__(256) prefix2_kernel(Segs S, float *aug2, int64_t d, double c, size_t stride,
                                                      bool lower32 = false) {
    const int64_t r = blockIdx.x;
    int64_t e4 = (int64_t)blockIdx.y * 256 + threadIdx.x;              // float4 index
    if (lower32) {
        // the consumer reads row i only up to the end of its 32-column block: threads cover those
        // entries only, row block rb (32 rows of 8 (rb + 1) float4 each) after the ones above it
        if (e4 >= lower32_count(d)) return;
        int rb = 0;
        while (128 * (int64_t)(rb + 1) * (rb + 2) <= e4) ++rb;
        const int64_t local = e4 - 128 * (int64_t)rb * (rb + 1);
        const int64_t w = 8 * (int64_t)(rb + 1);
        e4 = (rb * 32 + local / w) * (d / 4) + local % w;
    }
    if (e4 * 4 >= d * d) return;
    const int s0 = S.row_seg0[r], s1 = S.row_seg0[r + 1];
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int sb = s0; sb < s1; sb += 16) {
        const int cnt = min(16, s1 - sb);
        float4 g[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)                 // all loads in flight before the running sum
            if (q < cnt) g[q] = *reinterpret_cast<const float4 *>(aug2 + (size_t)(sb + q) * stride + 4 * e4);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            if (q < cnt) {
                *reinterpret_cast<float4 *>(aug2 + (size_t)(sb + q) * stride + 4 * e4) =
                    make_float4((float)(c * acc[0]), (float)(c * acc[1]), (float)(c * acc[2]), (float)(c * acc[3]));
                acc[0] += (double)g[q].x;
                acc[1] += (double)g[q].y;
                acc[2] += (double)g[q].z;
                acc[3] += (double)g[q].w;
            }
        }
    }
}

// ---------------------------------------------------------------- factor
template <int D>
struct FactorCfg {
    static constexpr int NT = 2 * D;
    static constexpr int PW = D >= 512 ? 32 : 64;
};

template <int D>
__global__ void __launch_bounds__(FactorCfg<D>::NT, 1) factor2_kernel(Segs S, float *aug2) {
    extern __shared__ float smf[];
    const int nseg = *S.nseg;
    for (int s = blockIdx.x; s < nseg; s += gridDim.x) {
        float *Ms = aug2 + (size_t)s * 2 * D * D;
        float4 *bot = reinterpret_cast<float4 *>(Ms + (size_t)D * D);     // appended block <- I
        for (int e = threadIdx.x; e < D * D / 4; e += FactorCfg<D>::NT) {
            const int i = (4 * e) / D, j = (4 * e) % D;
            bot[e] = make_float4(i == j, i == j + 1, i == j + 2, i == j + 3);
        }
        __syncthreads();
        pc::panel_chol<FactorCfg<D>::PW, FactorCfg<D>::NT>(Ms, D, 2 * D, D, true, nullptr, true, smf);
    }
}

// ---------------------------------------------------------------- A = B B^T
__device__ __forceinline__ void split3(float v, __nv_bfloat16 &h, __nv_bfloat16 &m, __nv_bfloat16 &l) {
    h = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(h);
    m = __float2bfloat16_rn(r1);
    l = __float2bfloat16_rn(r1 - __bfloat162float(m));
}

// A_nk = sum_{m >= max(n,k)} B_nm B_km (B upper triangular); 64 x 64 tiles,
// grid (segment, tile).
template <int D>
__global__ void __launch_bounds__(256) ainv_kernel(Segs S, const float *aug2, __nv_bfloat16 *A3) {
    const int s = blockIdx.x;
    if (s >= *S.nseg) return;
    constexpr int NTL = D / 64;
    const int I = blockIdx.y / NTL, J = blockIdx.y % NTL;
    const float *B = aug2 + (size_t)s * 2 * D * D + (size_t)D * D;
    __shared__ float As[32][65];
    __shared__ float Bs[32][65];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    const int m_start = (I > J ? I : J) * 64;
    for (int m0 = m_start; m0 < D; m0 += 32) {
        for (int e = tid; e < 64 * 32; e += 256) {
            const int rr = e >> 5, kk = e & 31;
            As[kk][rr] = B[(size_t)(I * 64 + rr) * D + m0 + kk];
            Bs[kk][rr] = B[(size_t)(J * 64 + rr) * D + m0 + kk];
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
    __nv_bfloat16 *A = A3 + (size_t)s * 3 * D * D;
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            __nv_bfloat16 h, m, l;
            split3(acc[q][r], h, m, l);
            const size_t o = (size_t)(I * 64 + ty * 4 + q) * D + J * 64 + tx * 4 + r;
            A[o] = h;
            A[(size_t)D * D + o] = m;
            A[(size_t)2 * D * D + o] = l;
        }
}

// ---------------------------------------------------------------- tcgen05 K-major GEMM core
// TMEM[128 x NTOT] (+)= sum over chunks c of A_c (128 x 64) B_c (NTOT x 64)^T.
// `load(c, a_saddr, b_saddr)` issues the cp.async fills of chunk c (K-major
// 128-byte swizzle); one thread issues the MMAs; NS stages in flight.
template <int NTOT, int NS, class Load>
__device__ __forceinline__ bool tc_gemm_kmajor(uint32_t tbase, int nchunks, uint32_t sbase, uint64_t *mbar,
                                               Load load, int32_t *st) {
    constexpr uint32_t A_BYTES = 128 * 128;
    constexpr uint32_t STAGE = A_BYTES + NTOT * 128;
    constexpr int NPER = NTOT < 256 ? NTOT : 256;
    constexpr int NMMA = NTOT / NPER;
    constexpr uint32_t idesc = tc::idesc_bf16(128, NPER, false, false);
    bool ok = true;
    for (int c = 0; c < NS - 1; ++c) {
        if (c < nchunks) load(c, sbase + (uint32_t)c * STAGE, sbase + (uint32_t)c * STAGE + A_BYTES);
        tc::cp_async_commit();
    }
    for (int c = 0; c < nchunks; ++c) {
        const int cn = c + NS - 1;
        if (cn < nchunks) {
            if (cn >= NS) ok &= tc::mbar_wait(&mbar[cn % NS], (uint32_t)((cn / NS) - 1) & 1u, st);
            const uint32_t sa = sbase + (uint32_t)(cn % NS) * STAGE;
            load(cn, sa, sa + A_BYTES);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<NS - 1>();
        tc::fence_async_smem();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc::fence_after_sync();
            const uint32_t sa = sbase + (uint32_t)(c % NS) * STAGE, sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = tc::sdesc(sa + kk * 32, 16, 1024);
#pragma unroll
                for (int nb = 0; nb < NMMA; ++nb) {
                    const uint64_t bd = tc::sdesc(sb + (uint32_t)nb * 256 * 128 + kk * 32, 16, 1024);
                    tc::mma_bf16(tbase + (uint32_t)(nb * 256), ad, bd, idesc, (c > 0 || kk > 0) ? 1u : 0u);
                }
            }
            tc::mma_commit(&mbar[c % NS]);
        }
        __syncthreads();
    }
    if (nchunks > 0) ok &= tc::mbar_wait(&mbar[(nchunks - 1) % NS], (uint32_t)((nchunks - 1) / NS) & 1u, st);
    ok = __syncthreads_and(ok) != 0;
    tc::fence_after_sync();
    return ok;
}

// cp.async fill of a K-major tile: `rows` rows of 64 bf16 from a row-major
// matrix (row pointer from `rowp(r)`, or zeros when it returns nullptr).
template <class RowPtr>
__device__ __forceinline__ void fill_kmajor(uint32_t saddr, int rows, RowPtr rowp) {
    for (int e = threadIdx.x; e < rows * 8; e += blockDim.x) {
        const int r = e >> 3, ch = e & 7;
        const __nv_bfloat16 *g = rowp(r);
        tc::cp_async16(saddr + tc::kmajor_off(r, ch * 8), g ? (const void *)(g + ch * 8) : (const void *)rowp(-1),
                       g ? 16u : 0u);
    }
}

template <int D>
struct VCfg {
    static constexpr int NS = D >= 512 ? 2 : 3;
    static constexpr uint32_t STAGE = 128 * 128 + D * 128;
    static constexpr size_t SMEM = NS * STAGE + 1024;
};

// V = X_s A_s (one 128-position block per CTA), written as three bf16 pieces.
template <int D>
__global__ void __launch_bounds__(128, 1) vgemm_kernel(const __nv_bfloat16 *__restrict__ H, Segs S,
                                                        const __nv_bfloat16 *__restrict__ A3,
                                                        __nv_bfloat16 *V3, int64_t N, float scale, int32_t *st) {
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[VCfg<D>::NS];
    __shared__ uint32_t tmem_base;
    const int s = blockIdx.x;
    if (s >= *S.nseg) return;
    const int len = S.len[s];
    const int mb = blockIdx.y;
    if (mb * 128 >= len) return;
    const int64_t start = S.start[s];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    if (warp == 0) tc::tmem_alloc(&tmem_base, D);
    if (tid == 0) {
        for (int i = 0; i < VCfg<D>::NS; ++i) tc::mbar_init(&mbar[i], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const __nv_bfloat16 *Xb = H + (start + (int64_t)mb * 128) * D;
    const int rows_valid = min(128, len - mb * 128);
    const __nv_bfloat16 *Aseg = A3 + (size_t)s * 3 * D * D;
    constexpr int KC = D / 64;
    auto load = [&](int c, uint32_t sa, uint32_t sb) {
        const int p = c / KC, kc = c % KC;
        fill_kmajor(sa, 128, [&](int r) -> const __nv_bfloat16 * {
            return r < 0 ? Xb : (r < rows_valid ? Xb + (int64_t)r * D + kc * 64 : nullptr);
        });
        const __nv_bfloat16 *Ap = Aseg + (size_t)p * D * D + kc * 64;
        fill_kmajor(sb, D, [&](int r) -> const __nv_bfloat16 * { return Ap + (int64_t)(r < 0 ? 0 : r) * D; });
    };
    const bool ok = tc_gemm_kmajor<D, VCfg<D>::NS>(tbase, 3 * KC, base, mbar, load, st);
    if (ok) {
        // per 64-column block: TMEM -> three bf16 pieces in shared memory (row-major, 144-byte
        // rows, reusing the stage buffers) -> whole 128-byte row segments to V3
        tc::cp_async_wait<0>();
        __syncthreads();
        uint8_t *stg = smraw + (base - tc::smem_u32(smraw));
        constexpr int RS = 144;
        const int row = warp * 32 + lane;
        __nv_bfloat16 *vb = V3 + (size_t)(start + mb * 128) * D;
#pragma unroll 1
        for (int cb = 0; cb < D; cb += 64) {
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                float v[16];
                tc::tmem_ld16(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)(cb + 16 * j), v);
                __align__(16) __nv_bfloat16 h[16], m[16], l[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) split3(scale * v[i], h[i], m[i], l[i]);
#pragma unroll
                for (int p = 0; p < 3; ++p) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(p == 0 ? h : (p == 1 ? m : l));
                    uint4 *d = reinterpret_cast<uint4 *>(stg + (size_t)(p * 128 + row) * RS + j * 32);
                    d[0] = src[0];
                    d[1] = src[1];
                }
            }
            __syncthreads();
            for (int e = tid; e < 3 * 128 * 8; e += 128) {
                const int pr = e >> 3, ch = e & 7, p = pr >> 7, r = pr & 127;
                if (r < rows_valid)
                    *reinterpret_cast<uint4 *>(vb + (size_t)p * N * D + (size_t)r * D + cb + ch * 8) =
                        *reinterpret_cast<const uint4 *>(stg + (size_t)pr * RS + ch * 16);
            }
            __syncthreads();
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, D);
}

struct KCfg {
    static constexpr int NS = 4;
    static constexpr uint32_t STAGE = 128 * 128 + 128 * 128;
    static constexpr size_t SMEM = NS * STAGE + 1024;
};

// G'_s = c X_s V^T on the lower 128 x 128 blocks of the segment; grid (segment, 10).
template <int D>
__global__ void __launch_bounds__(128, 1) kgemm_kernel(const __nv_bfloat16 *__restrict__ H, Segs S,
                                                        const __nv_bfloat16 *__restrict__ V3, int64_t N,
                                                        float c_rate, float *gp, int32_t *st) {
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[KCfg::NS];
    __shared__ uint32_t tmem_base;
    const int s = blockIdx.x;
    if (s >= *S.nseg) return;
    const int t = blockIdx.y;
    int mi = 0;
    while ((mi + 1) * (mi + 2) / 2 <= t) ++mi;
    const int nj = t - mi * (mi + 1) / 2;
    const int len = S.len[s];
    if (mi * 128 >= len) return;
    const int64_t start = S.start[s];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = (tc::smem_u32(smraw) + 1023u) & ~1023u;
    if (warp == 0) tc::tmem_alloc(&tmem_base, 128);
    if (tid == 0) {
        for (int i = 0; i < KCfg::NS; ++i) tc::mbar_init(&mbar[i], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const int rows_a = min(128, len - mi * 128), rows_b = min(128, len - nj * 128);
    const __nv_bfloat16 *Xa = H + (start + (int64_t)mi * 128) * D;
    const __nv_bfloat16 *Vb = V3 + (size_t)(start + nj * 128) * D;
    constexpr int KC = D / 64;
    auto load = [&](int c, uint32_t sa, uint32_t sb) {
        const int p = c / KC, kc = c % KC;
        fill_kmajor(sa, 128, [&](int r) -> const __nv_bfloat16 * {
            return r < 0 ? Xa : (r < rows_a ? Xa + (int64_t)r * D + kc * 64 : nullptr);
        });
        const __nv_bfloat16 *Vp = Vb + (size_t)p * N * D;
        fill_kmajor(sb, 128, [&](int r) -> const __nv_bfloat16 * {
            return r < 0 ? Vp : (r < rows_b ? Vp + (int64_t)r * D + kc * 64 : nullptr);
        });
    };
    const bool ok = tc_gemm_kmajor<128, KCfg::NS>(tbase, 3 * KC, base, mbar, load, st);
    if (ok) {
        const int i = mi * 128 + warp * 32 + lane;
        const int ld = ldg_of(len);
        float *G = gp + (size_t)start * kSegMax + (size_t)i * ld + nj * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
            if (i < len) {
                const int j0 = nj * 128 + c0;
                if (j0 + 16 <= len) {
                    float4 *dst = reinterpret_cast<float4 *>(G + c0);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_float4(c_rate * v[4 * q], c_rate * v[4 * q + 1], c_rate * v[4 * q + 2],
                                             c_rate * v[4 * q + 3]);
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (j0 + q < len) G[c0 + q] = c_rate * v[q];
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 128);
}

// ---------------------------------------------------------------- in-segment Cholesky
constexpr int kInsegPW = 64, kInsegNT = 512;

__global__ void __launch_bounds__(kInsegNT, 1) inseg_kernel(Segs S, float *gp, float *dR) {
    extern __shared__ float smi[];
    const int nseg = *S.nseg;
    for (int s = blockIdx.x; s < nseg; s += gridDim.x) {
        const int len = S.len[s];
        const int64_t start = S.start[s];
        pc::panel_chol<kInsegPW, kInsegNT>(gp + (size_t)start * kSegMax, ldg_of(len), len, len, false,
                                           dR + start, false, smi);
    }
}

template <int D>
dbc_status run_tc(const __nv_bfloat16 *H, const int64_t *offsets, int64_t rows, int64_t T, int64_t N,
                  float eps2, float *dR, const Layout2 &L, int32_t *st, cudaStream_t stream) {
    const double c = (double)D / (double)eps2;
    const int64_t ns = nseg_upper(rows, N);
    const int sms = num_sms();
    seg_table_kernel<<<1, 1024, 0, stream>>>(offsets, rows, T, N, ns, kSegMax, L.segs, st);
    launch_gram_tc<D>(H, ns, L.segs, L.aug2, (size_t)2 * D * D, st, stream);
    prefix2_kernel<<<dim3((unsigned)rows, (unsigned)((D * D / 4 + 255) / 256)), 256, 0, stream>>>(
        L.segs, L.aug2, D, c, (size_t)2 * D * D);
    using F = FactorCfg<D>;
    using PF = pc::PanelChol<F::PW, F::NT>;
    cudaFuncSetAttribute(factor2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PF::SMEM);
    const int grid_seg = (int)std::min<int64_t>(ns, (int64_t)sms * 8);
    factor2_kernel<D><<<grid_seg, F::NT, PF::SMEM, stream>>>(L.segs, L.aug2);
    ainv_kernel<D><<<dim3((unsigned)ns, (unsigned)((D / 64) * (D / 64))), 256, 0, stream>>>(L.segs, L.aug2, L.A3);
    cudaFuncSetAttribute(vgemm_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)VCfg<D>::SMEM);
    vgemm_kernel<D><<<dim3((unsigned)ns, 4), 128, VCfg<D>::SMEM, stream>>>(H, L.segs, L.A3, L.V3, N, 1.f, st);
    cudaFuncSetAttribute(kgemm_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KCfg::SMEM);
    kgemm_kernel<D><<<dim3((unsigned)ns, 10), 128, KCfg::SMEM, stream>>>(H, L.segs, L.V3, N, (float)c, L.gp, st);
    using PI = pc::PanelChol<kInsegPW, kInsegNT>;
    cudaFuncSetAttribute(inseg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PI::SMEM);
    inseg_kernel<<<grid_seg, kInsegNT, PI::SMEM, stream>>>(L.segs, L.gp, dR);
    count_launches(9);
    return launch_status();
}

// ================================================================ d = 256: TMEM-resident factorizations
// Segments of at most 256 positions: the start state's factorization with its
// inverse factor B = L^{-T} (FACTOR) and the in-segment Cholesky (INSEG) each
// run inside one SM's tensor memory; the whitening Y = sqrt(c) X B in between.
constexpr int kLmaxTmem = 256;

struct Layout3 {
    Segs segs;
    float *P;               // per segment: [D][D] Gram -> c-scaled prefix
    __nv_bfloat16 *Bscr;    // per segment: [3][D][D] pieces of B = L^{-T} (rows below a panel unstored)
    size_t bytes;
};

// ns_given >= 0: exactly that many segments (the streaming continuation), else
// the batch upper bound.
inline Layout3 carve3(void *ws, int64_t rows, int64_t N, int64_t d, int64_t ns_given = -1) {
    Carver c(ws);
    const int64_t ns = ns_given >= 0 ? ns_given : nseg_upper(rows, N, kLmaxTmem);
    Layout3 L;
    L.segs.start = c.take<int64_t>(ns);
    L.segs.len = c.take<int32_t>(ns);
    L.segs.row = c.take<int32_t>(ns);
    L.segs.k = c.take<int32_t>(ns);
    L.segs.row_seg0 = c.take<int32_t>(rows + 1);
    L.segs.nseg = c.take<int32_t>(1);
    L.P = c.take<float>((size_t)ns * d * d);
    L.Bscr = c.take<__nv_bfloat16>((size_t)ns * 3 * d * d);
    L.bytes = c.off;
    return L;
}

}  // namespace cr
}  // namespace dbc

#include "tmem_chol.cuh"
#include "gram_prefix.cuh"
#include "gram_tma.cuh"
#include "tma_host.cuh"

namespace dbc {
namespace cr {

// P_s = c (state + the row's earlier segment Grams) for every segment, through the fused TMA-fed
// Gram + prefix kernel (one CTA per row and 128 x 64 tile).  Returns false (nothing
// launched) when the row count and lengths favour the segment-parallel Gram and prefix kernels,
// or when no tensor map can be encoded.
inline bool launch_gram_prefix(const __nv_bfloat16 *H, int64_t N, int64_t rows, int64_t ns, const Segs &segs,
                               float *P, double *state, double c, int32_t *st, cudaStream_t stream) {
    const int sms = num_sms();
    // Each CTA walks its row's segments one after another (about 3 us a segment), so with fewer
    // CTAs than half the SMs the segment-parallel Gram kernel and the prefix kernel finish first
    // (8 rows of 8192 positions: 61 us against 100 us; 64 rows of 4096: 252 us against 158 us).
    if (rows * GramPrefixCfg<64>::TILES * 2 < sms && ns > rows * 2) return false;
    if (rows * 6 > INT32_MAX / 2) return false;
    CUtensorMap tm;
    if (!tma::encode_bf16_rows(&tm, H, (uint64_t)N, 256, 64)) return false;
    // 128 x 64 tiles: 32 running sums per epilogue thread (wider tiles would spill registers)
    using C = GramPrefixCfg<64>;
    cudaFuncSetAttribute(gram_prefix_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    gram_prefix_kernel<64><<<(unsigned)(rows * C::TILES), C::NT, C::SMEM, stream>>>(tm, segs, rows, P, state, c, st);
    return true;
}

// The factor and in-segment Cholesky launches of ns segments (tensor maps over P and B's pieces for the
// factor mode's TMA loads and stores).  False (nothing launched) when a tensor map cannot be encoded.
inline bool launch_tmem_chol(const __nv_bfloat16 *H, int64_t N, int64_t ns, const Layout3 &L, float c, float *dR,
                             int32_t *st, cudaStream_t stream) {
    constexpr int D = 256;
    CUtensorMap tmP, tmB, tmX;
    if (!tma::encode_f32_rows(&tmP, L.P, (uint64_t)ns * D, D, 32)) return false;
    if (!tma::encode_bf16_rows(&tmB, L.Bscr, (uint64_t)ns * 3 * D, D, 64)) return false;
    const int xbox = (int)std::min<int64_t>(N, 256);
    if (!tma::encode_bf16_rows(&tmX, H, (uint64_t)N, D, (uint32_t)xbox)) return false;
    const int grid = (int)std::min<int64_t>(ns, (int64_t)num_sms());
    cudaFuncSetAttribute(tmem_chol_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TmemChol::SMEM);
    cudaFuncSetAttribute(tmem_chol_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TmemChol::SMEM);
    tmem_chol_kernel<true><<<grid, TmemChol::NT, TmemChol::SMEM, stream>>>(tmP, tmB, tmX, xbox, L.segs, L.P, L.Bscr, nullptr,
                                                                         N, c, dR, st);
    tmem_chol_kernel<false><<<grid, TmemChol::NT, TmemChol::SMEM, stream>>>(tmP, tmB, tmX, xbox, L.segs, nullptr, L.Bscr, H,
                                                                          N, c, dR, st);
    return true;
}

inline dbc_status run_tmem(const __nv_bfloat16 *H, const int64_t *offsets, int64_t rows, int64_t T, int64_t N,
                           float eps2, float *dR, const Layout3 &L, int32_t *st, cudaStream_t stream) {
    constexpr int D = 256;
    const double c = (double)D / (double)eps2;
    const int64_t ns = nseg_upper(rows, N, kLmaxTmem);
    seg_table_kernel<<<1, 1024, 0, stream>>>(offsets, rows, T, N, ns, kLmaxTmem, L.segs, st);
    const bool fused = launch_gram_prefix(H, N, rows, ns, L.segs, L.P, nullptr, c, st, stream);
    if (!fused) {
        // the factor kernel reads each row of P_s up to the end of its 32-column block only
        CUtensorMap tmH, tmG;
        if (tma::encode_bf16_rows(&tmH, H, (uint64_t)N, D, 64) &&
            tma::encode_f32_rows(&tmG, L.P, (uint64_t)ns * D, D, 128)) {
            cudaFuncSetAttribute(gram_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GramTma::SMEM);
            gram_tma_kernel<<<(unsigned)ns, 256, GramTma::SMEM, stream>>>(tmH, tmG, L.segs, st);
        } else {
            launch_gram_tc<D>(H, ns, L.segs, L.P, (size_t)D * D, st, stream, true);
        }
        prefix2_kernel<<<dim3((unsigned)rows, (unsigned)((lower32_count(D) + 255) / 256)), 256, 0, stream>>>(
            L.segs, L.P, D, c, (size_t)D * D, true);
    }
    if (!launch_tmem_chol(H, N, ns, L, (float)c, dR, st, stream)) return DBC_ERR_CUDA;
    count_launches(fused ? 4 : 5);
    return launch_status();
}

// ================================================================ streaming continuation (d = 256)
// `streams` rows of n new positions each continue streams that have already
// consumed t0 positions; their Gram sums S (float64, [streams][D][D], the
// caller's buffer) are the start state and are advanced by the new block.  The
// new positions are cut at the same absolute segment boundaries as a whole
// sequence (0, 64, 128, then every multiple of 256), so a segment is never
// longer than the prefix before it, and the values equal the whole sequence's.

// First boundary above t0 (index k1) and the number of pieces of [t0, t0 + n).
inline void stream_pieces(int64_t t0, int64_t n, int64_t &k1, int64_t &cnt) {
    const int k0 = seg_k0(kLmaxTmem);
    if (t0 < seg_bound(k0, kLmaxTmem)) {
        k1 = 0;
        while (seg_bound(k1, kLmaxTmem) <= t0) ++k1;
    } else {
        k1 = k0 + t0 / kLmaxTmem;           // seg_bound(k) = 256 (k - k0 + 1) > t0
    }
    cnt = n > 0 ? 1 : 0;
    while (n > 0 && seg_bound(k1 + cnt - 1, kLmaxTmem) < t0 + n) ++cnt;
}

__global__ void __launch_bounds__(256) stream_seg_table_kernel(int64_t streams, int64_t n, int64_t t0, int64_t k1,
                                                               int64_t cnt, Segs S) {
    const int64_t total = streams * cnt;
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < total; s += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = s / cnt, j = s - r * cnt;
        const int64_t a = j == 0 ? t0 : seg_bound(k1 + j - 1, kLmaxTmem);
        const int64_t e = j + 1 < cnt ? seg_bound(k1 + j, kLmaxTmem) : t0 + n;
        S.start[s] = r * n + (a - t0);
        S.len[s] = (int32_t)(e - a);
        S.row[s] = (int32_t)r;
        S.k[s] = (int32_t)j;
        if (j == 0) S.row_seg0[r] = (int32_t)s;
        if (s == 0) {
            S.row_seg0[streams] = (int32_t)total;
            *S.nseg = (int32_t)total;
        }
    }
}

// P_s = c (S_row + sum of the row's earlier segment Grams), running sums in
// float64 starting from the carried state, which is advanced to the end.
__global__ void __launch_bounds__(256) prefix_stream_kernel(Segs S, float *P, double *state, int64_t d, double c) {
    const int64_t r = blockIdx.x;
    const int64_t e4 = (int64_t)blockIdx.y * 256 + threadIdx.x;        // float4 index
    if (e4 * 4 >= d * d) return;
    double *sr = state + (size_t)r * d * d + 4 * e4;
    double acc[4] = {sr[0], sr[1], sr[2], sr[3]};
    const int s0 = S.row_seg0[r], s1 = S.row_seg0[r + 1];
    for (int sb = s0; sb < s1; sb += 16) {
        const int cnt = min(16, s1 - sb);
        float4 g[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
            if (q < cnt) g[q] = *reinterpret_cast<const float4 *>(P + (size_t)(sb + q) * d * d + 4 * e4);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            if (q < cnt) {
                *reinterpret_cast<float4 *>(P + (size_t)(sb + q) * d * d + 4 * e4) =
                    make_float4((float)(c * acc[0]), (float)(c * acc[1]), (float)(c * acc[2]), (float)(c * acc[3]));
                acc[0] += (double)g[q].x;
                acc[1] += (double)g[q].y;
                acc[2] += (double)g[q].z;
                acc[3] += (double)g[q].w;
            }
        }
    }
    sr[0] = acc[0]; sr[1] = acc[1]; sr[2] = acc[2]; sr[3] = acc[3];
}

inline dbc_status run_tmem_stream(const __nv_bfloat16 *H, int64_t streams, int64_t n, int64_t t0, int64_t k1,
                                  int64_t cnt, float eps2, double *state, float *dR, const Layout3 &L, int32_t *st,
                                  cudaStream_t stream) {
    constexpr int D = 256;
    const double c = (double)D / (double)eps2;
    const int64_t ns = streams * cnt;
    const int64_t N = streams * n;
    const int sms = num_sms();
    const int tgrid = (int)std::max<int64_t>(1, std::min<int64_t>((ns + 255) / 256, (int64_t)sms * 4));
    stream_seg_table_kernel<<<tgrid, 256, 0, stream>>>(streams, n, t0, k1, cnt, L.segs);
    const bool fused = launch_gram_prefix(H, N, streams, ns, L.segs, L.P, state, c, st, stream);
    if (!fused) {
        launch_gram_tc<D>(H, ns, L.segs, L.P, (size_t)D * D, st, stream);
        prefix_stream_kernel<<<dim3((unsigned)streams, (unsigned)((D * D / 4 + 255) / 256)), 256, 0, stream>>>(
            L.segs, L.P, state, D, c);
    }
    if (!launch_tmem_chol(H, N, ns, L, (float)c, dR, st, stream)) return DBC_ERR_CUDA;
    count_launches(fused ? 4 : 5);
    return launch_status();
}

}  // namespace cr
}  // namespace dbc
