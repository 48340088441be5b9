// chunk_coding_rate: marginal lossy coding rate dR_t of every byte position.
//
// Method (ByteFlow, arXiv 2603.03583; paper.rainbus.top summary,
// "Prerequisites: lossy coding rate" and "Method steps", stage 2):
//   R_eps(H) = 1/2 logdet(I + c H H^T), c = d/eps^2,  dR_t = R(h_0..t) - R(h_0..t-1).
// Sylvester's identity turns the T x T determinant into a d x d one and the
// matrix determinant lemma gives dR_t = 1/2 log(1 + c h_t^T M_{t-1}^{-1} h_t),
// M_t = I + c sum_{i<=t} h_i h_i^T.
//
// Segment-parallel evaluation (all segments of all rows are independent
// except for an exclusive prefix of their Grams):
//   1. every row is cut into segments [0,64) [64,128) [128,256) [256,512) and
//      then 512-long pieces;
//   2. gram:   G_s = X_s^T X_s for every segment (bf16 products are exact,
//              fp32 accumulation);
//   3. prefix: P_s = c sum_{s' < s} G_s' (float64 running sum, stored fp32);
//              M_s = I + P_s is the state at the segment start;
//   4. factor: Cholesky of M_s carried on the augmented matrix [P_s ; X_s]
//              with the identity kept implicit: the first d columns give
//              L_s (L_s L_s^T = M_s) and, in the rows below, Y_s = X_s L_s^{-T};
//   5. ygram:  G'_s = c Y_s Y_s^T (in-segment Gram in the whitened frame);
//   6. in-segment Cholesky of I + G'_s with the identity implicit: by the
//      Schur complement the squared diagonal of the factor at position t is
//      1 + c h_t^T M_{t-1}^{-1} h_t, so the carried excess e_t (diagonal minus
//      the implicit 1) gives dR_t = 1/2 log1p(e_t) without rounding the 1.
//   The first segment of each row (M = I) has the largest cancellation and
//   is done entirely in float64 (G' = c X X^T, Cholesky, log1p).
#include <math.h>

#include "common.cuh"
#include "tc.cuh"

namespace dbc {
namespace cr {

constexpr int PW = 32;          // Cholesky panel width
constexpr int kSegMax = 512;    // longest segment

// Segment boundaries of a row: 0, 64, 128, then (lmax = 512) 256 and every
// multiple of 512, or (lmax = 256) every multiple of 256.  Lengths double
// until lmax so a segment is never longer than the prefix before it.
__host__ __device__ inline int seg_k0(int lmax) { return lmax >= 512 ? 4 : 3; }

__host__ __device__ inline int64_t seg_bound(int64_t k, int lmax) {
    const int k0 = seg_k0(lmax);
    if (k < k0) return k == 0 ? 0 : (k == 1 ? 64 : (k == 2 ? 128 : 256));
    return (int64_t)lmax * (k - k0 + 1);
}

__host__ __device__ inline int64_t seg_count(int64_t n, int lmax) {
    if (n <= 0) return 0;
    const int k0 = seg_k0(lmax);
    int64_t c = 0;
    for (int k = 0; k < k0; ++k) c += seg_bound(k, lmax) < n;
    if (n > lmax) c += (n - 1) / lmax;
    return c;
}

inline int64_t nseg_upper(int64_t rows, int64_t N, int lmax = kSegMax) {
    return (int64_t)seg_k0(lmax) * rows + N / lmax + 1;
}

struct Segs {
    int64_t *start;      // absolute first position
    int32_t *len;        // positions in the segment
    int32_t *row;        // owning row
    int32_t *k;          // index of the segment inside its row
    int32_t *row_seg0;   // [rows+1] first segment of each row
    int32_t *nseg;       // number of segments (device)
};

struct Layout {
    Segs segs;
    float *aug;          // per segment: (d + kSegMax) x d
    float *gp;           // per segment at start*kSegMax: len x len
    size_t bytes;
};

inline Layout carve(void *ws, int64_t rows, int64_t N, int64_t d) {
    Carver c(ws);
    const int64_t ns = nseg_upper(rows, N);
    Layout L;
    L.segs.start = c.take<int64_t>(ns);
    L.segs.len = c.take<int32_t>(ns);
    L.segs.row = c.take<int32_t>(ns);
    L.segs.k = c.take<int32_t>(ns);
    L.segs.row_seg0 = c.take<int32_t>(rows + 1);
    L.segs.nseg = c.take<int32_t>(1);
    L.aug = c.take<float>((size_t)ns * (size_t)(d + kSegMax) * (size_t)d);
    L.gp = c.take<float>((size_t)N * kSegMax + 1);
    L.bytes = c.off;
    return L;
}

// ---------------------------------------------------------------- seg table
__global__ void __launch_bounds__(1024) seg_table_kernel(const int64_t *offsets, int64_t rows,
                                                         int64_t T, int64_t N, int64_t ns, int lmax, Segs S,
                                                         int32_t *st) {
    __shared__ int64_t wsum[32];
    __shared__ int64_t carry;
    __shared__ int64_t sh_excl[1024], sh_a[1024], sh_n[1024], sh_cnt[1024];   // per row of the current block
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int64_t base = 0; base < rows; base += blockDim.x) {
        const int64_t r = base + tid;
        int64_t a = 0, n = 0, cnt = 0;
        if (r < rows) {
            row_bounds(offsets, r, T, a, n);
            if (a < 0 || n < 0 || a + n > N) {   // malformed offsets: treat the row as empty
                flag(st, DBC_ERR_BOUNDS);
                n = 0;
            }
            cnt = seg_count(n, lmax);
        }
        int64_t x = cnt;
        for (int o = 1; o < 32; o <<= 1) {
            int64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int64_t w = (lane < (int)(blockDim.x >> 5)) ? wsum[lane] : 0;
            for (int o = 1; o < 32; o <<= 1) {
                int64_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            wsum[lane] = w;
        }
        __syncthreads();
        const int64_t excl = carry + (wid ? wsum[wid - 1] : 0) + x - cnt;
        if (r < rows) S.row_seg0[r] = (int32_t)excl;
        sh_excl[tid] = excl;
        sh_a[tid] = a;
        sh_n[tid] = n;
        sh_cnt[tid] = cnt;
        __syncthreads();
        // the entries: warp w fills the rows w, w + 32, ... of this block of rows, a lane per segment
        for (int rr = wid; rr < (int)blockDim.x && base + rr < rows; rr += (int)(blockDim.x >> 5)) {
            const int64_t e0 = sh_excl[rr], a0 = sh_a[rr], n0 = sh_n[rr], c0 = sh_cnt[rr];
            for (int64_t k = lane; k < c0 && e0 + k < ns; k += 32) {
                const int64_t s0 = seg_bound(k, lmax);
                const int64_t s1 = min(n0, seg_bound(k + 1, lmax));
                const int64_t s = e0 + k;
                S.start[s] = a0 + s0;
                S.len[s] = (int32_t)(s1 - s0);
                S.row[s] = (int32_t)(base + rr);
                S.k[s] = (int32_t)k;
            }
        }
        __syncthreads();
        if (tid == (int)blockDim.x - 1) carry = excl + cnt;
        __syncthreads();
    }
    if (tid == 0) {
        if (carry > ns) {
            flag(st, DBC_ERR_BOUNDS);
            carry = ns;
        }
        S.row_seg0[rows] = (int32_t)carry;
        *S.nseg = (int32_t)carry;
    }
}

// ---------------------------------------------------------------- gram
// G_s tile (64 x 64) = sum_t X[t, I-block]^T X[t, J-block]; grid (seg, tile).
template <class IN>
__global__ void __launch_bounds__(256) gram_kernel(const IN *__restrict__ H, int64_t d, Segs S,
                                                   float *aug, int32_t *st) {
    const int s = blockIdx.x;
    if (s >= *S.nseg) return;
    const int nt = (int)(d / 64);
    const int I = blockIdx.y / nt, J = blockIdx.y % nt;
    const int64_t start = S.start[s];
    const int len = S.len[s];
    __shared__ float As[32][64];
    __shared__ float Bs[32][64];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    bool bad = false;
    for (int t0 = 0; t0 < len; t0 += 32) {
        for (int e = tid; e < 32 * 64; e += 256) {
            const int tt = e >> 6, cc = e & 63;
            float va = 0.f, vb = 0.f;
            if (t0 + tt < len) {
                const IN *row = H + (start + t0 + tt) * d;
                va = ld_f(row + I * 64 + cc);
                vb = ld_f(row + J * 64 + cc);
                if (J == 0 && !isfinite(va)) bad = true;
            }
            As[tt][cc] = va;
            Bs[tt][cc] = vb;
        }
        __syncthreads();
#pragma unroll 8
        for (int tt = 0; tt < 32; ++tt) {
            float a[4], b[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) { a[q] = As[tt][ty * 4 + q]; b[q] = Bs[tt][tx * 4 + q]; }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[q][r] = fmaf(a[q], b[r], acc[q][r]);
        }
        __syncthreads();
    }
    if (bad) flag(st, DBC_ERR_NONFINITE);
    float *G = aug + (size_t)s * (size_t)(d + kSegMax) * (size_t)d;
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int r = 0; r < 4; ++r)
            G[(size_t)(I * 64 + ty * 4 + q) * d + J * 64 + tx * 4 + r] = acc[q][r];
}

// ---------------------------------------------------------------- gram (tensor cores)
// G_s = X_s^T X_s on tcgen05 (bf16 x bf16 products are exact, fp32 accumulation
// in TMEM).  A 64-position chunk of X_s is staged once in shared memory as an
// MN-major 128-byte-swizzled tile and read as both operands (A = features of
// this CTA's 128-row blocks, B = all d features).  Three stages keep the next
// cp.async fills in flight while the tensor core works on the current chunk.
// grid (segment, row-block group), 128 threads.
template <int D>
struct GramTC {
    static constexpr int NMB = (D == 256) ? 2 : 1;       // 128-row blocks per CTA
    static constexpr int GROUPS = (D / 128) / NMB;       // CTAs per segment
    static constexpr int NCOLS = NMB * D;                // TMEM columns used
    static constexpr int TMEM_COLS = NCOLS <= 128 ? 128 : (NCOLS <= 256 ? 256 : 512);
    static constexpr int KC = 64;                        // positions per chunk
    static constexpr uint32_t LBO = KC * 128;            // bytes of one 64-feature block
    static constexpr uint32_t STAGE = (D / 64) * LBO;
    static constexpr int NS = 3;
    static constexpr size_t SMEM = NS * STAGE + 1024;
};

template <int D>
__global__ void __launch_bounds__(256, 1) gram_tc_kernel(const __nv_bfloat16 *__restrict__ H, Segs S,
                                                          float *aug, size_t mat_stride, bool lower, int32_t *st) {
    using C = GramTC<D>;
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar[C::NS];
    __shared__ uint32_t tmem_base;
    const int s = blockIdx.x;
    if (s >= *S.nseg) return;
    const int mb0 = blockIdx.y * C::NMB;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int len = S.len[s];
    const int64_t start = S.start[s];
    const uint32_t raw = tc::smem_u32(smraw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    if (warp == 0) tc::tmem_alloc(&tmem_base, C::TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < C::NS; ++i) tc::mbar_init(&mbar[i], 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = tmem_base;
    const int nchunks = (len + C::KC - 1) / C::KC;
    constexpr int F8 = D / 8;                            // 16-byte groups per position

    auto load = [&](int c) {
        const uint32_t sb = base + (uint32_t)(c % C::NS) * C::STAGE;
        const int t0 = c * C::KC;
        for (int e = tid; e < C::KC * F8; e += 256) {
            const int p = e / F8, f8 = e - (e / F8) * F8;
            const int pos = t0 + p;
            const __nv_bfloat16 *src = H + (start + (pos < len ? pos : 0)) * D + f8 * 8;
            tc::cp_async16(sb + tc::mnmajor_off(f8 * 8, p, C::LBO), src, pos < len ? 16u : 0u);
        }
        tc::cp_async_commit();
    };

    bool ok = true;
    for (int c = 0; c < C::NS - 1; ++c) {
        if (c < nchunks) load(c); else tc::cp_async_commit();
    }
    constexpr uint32_t idesc = tc::idesc_bf16(128, D < 256 ? D : 256, true, true);
    // lower: the first 128-row block only needs its first 128 columns (D = 256 with two row blocks)
    constexpr uint32_t idesc_half = tc::idesc_bf16(128, 128, true, true);
    const bool half0 = lower && D == 256 && C::NMB == 2;
    for (int c = 0; c < nchunks; ++c) {
        const int cn = c + C::NS - 1;
        if (cn < nchunks) {
            if (cn >= C::NS) ok &= tc::mbar_wait(&mbar[cn % C::NS], (uint32_t)((cn / C::NS) - 1) & 1u, st);
            load(cn);
        } else {
            tc::cp_async_commit();
        }
        tc::cp_async_wait<C::NS - 1>();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t sb = base + (uint32_t)(c % C::NS) * C::STAGE;
#pragma unroll
            for (int kk = 0; kk < C::KC / 16; ++kk) {
#pragma unroll
                for (int m = 0; m < C::NMB; ++m) {
                    const uint64_t ad = tc::sdesc(sb + (uint32_t)(2 * (mb0 + m)) * C::LBO + kk * 2048, C::LBO, 1024);
#pragma unroll
                    for (int nb = 0; nb < (D + 255) / 256; ++nb) {
                        const uint64_t bd = tc::sdesc(sb + (uint32_t)(4 * nb) * C::LBO + kk * 2048, C::LBO, 1024);
                        tc::mma_bf16(tbase + (uint32_t)(m * D + nb * 256), ad, bd,
                                     (half0 && m == 0) ? idesc_half : idesc, (c > 0 || kk > 0) ? 1u : 0u);
                    }
                }
            }
            tc::mma_commit(&mbar[c % C::NS]);
        }
        __syncthreads();
    }
    if (nchunks > 0) ok &= tc::mbar_wait(&mbar[(nchunks - 1) % C::NS], (uint32_t)((nchunks - 1) / C::NS) & 1u, st);
    ok = __syncthreads_and(ok) != 0;      // the warp-collective TMEM loads below need a uniform decision
    tc::fence_after_sync();
    float *G = aug + (size_t)s * mat_stride;
    bool bad = false;
    if (ok) {
        // 8 warps: warps w and w + 4 share the TMEM lanes of group w % 4 and take either one
        // row block each (two blocks) or one half of the columns each (one block)
        const int slot = warp >> 2, lg = warp & 3;
        const int m = C::NMB == 2 ? slot : 0;
        const int cbeg = C::NMB == 2 ? 0 : slot * (D / 2);
        const int cend = C::NMB == 2 ? ((half0 && m == 0) ? 128 : D) : cbeg + D / 2;
        {
            const int row = (mb0 + m) * 128 + lg * 32 + lane;
#pragma unroll 1
            for (int c0 = cbeg; c0 < cend; c0 += 16) {
                float v[16];
                tc::tmem_ld16(tbase + ((uint32_t)(lg * 32) << 16) + (uint32_t)(m * D + c0), v);
                if (nchunks == 0) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (row == c0 + i) bad |= !isfinite(v[i]);
                float4 *dst = reinterpret_cast<float4 *>(G + (size_t)row * D + c0);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    }
    if (bad) flag(st, DBC_ERR_NONFINITE);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, C::TMEM_COLS);
}

// ---------------------------------------------------------------- prefix
// In place over each row's segments: G_s -> P_s = c * sum_{s'<s} G_s' (fp64 sum).
__global__ void __launch_bounds__(256) prefix_kernel(Segs S, float *aug, int64_t d, double c) {
    const int64_t r = blockIdx.x;
    const int64_t e = (int64_t)blockIdx.y * 256 + threadIdx.x;
    if (e >= d * d) return;
    const int s0 = S.row_seg0[r], s1 = S.row_seg0[r + 1];
    const size_t stride = (size_t)(d + kSegMax) * (size_t)d;
    double acc = 0.0;
    for (int s = s0; s < s1; ++s) {
        float *p = aug + (size_t)s * stride + e;
        const float g = *p;
        *p = (float)(c * acc);
        acc += (double)g;
    }
}

// Rows d .. d+len-1 of the augmented matrix receive X_s (fp32).
template <class IN>
__global__ void __launch_bounds__(256) fill_x_kernel(const IN *__restrict__ H, int64_t d, Segs S,
                                                     float *aug) {
    const int s = blockIdx.x;
    if (s >= *S.nseg || S.k[s] == 0) return;
    const int64_t start = S.start[s];
    const int64_t cnt = (int64_t)S.len[s] * d;
    float *dst = aug + (size_t)s * (size_t)(d + kSegMax) * (size_t)d + (size_t)d * d;
    for (int64_t e = (int64_t)blockIdx.y * 256 + threadIdx.x; e < cnt; e += (int64_t)gridDim.y * 256)
        dst[e] = ld_f(H + start * d + e);
}

// ---------------------------------------------------------------- Cholesky
// Right-looking panel Cholesky of I + A with the identity implicit, on the
// first `ncols` columns of an nrows x ncols row-major block (lower part).
// The diagonal value met when a column is factored is the excess e (Schur
// complement minus 1); the stored diagonal becomes sqrt(1 + e).
// FACTOR: A = [P_s ; X_s] -> [L_s ; Y_s].  INSEG: A = G'_s -> dR = log1p(e)/2.
template <bool INSEG>
__global__ void __launch_bounds__(256) chol_kernel(Segs S, float *aug, float *gp, int64_t d,
                                                   float *dR) {
    extern __shared__ float P[];
    constexpr int LDP = PW + 1;
    const int tid = threadIdx.x;
    const int nseg = *S.nseg;
    for (int s = blockIdx.x; s < nseg; s += gridDim.x) {
        if (S.k[s] == 0) continue;
        const int len = S.len[s];
        const int64_t start = S.start[s];
        float *A;
        int ld, nrows, ncols;
        if (INSEG) {
            A = gp + (size_t)start * kSegMax;
            ld = len; nrows = len; ncols = len;
        } else {
            A = aug + (size_t)s * (size_t)(d + kSegMax) * (size_t)d;
            ld = (int)d; nrows = (int)d + len; ncols = (int)d;
        }
        for (int j0 = 0; j0 < ncols; j0 += PW) {
            const int nb = min(PW, ncols - j0);
            const int m = nrows - j0;
            for (int e = tid; e < m * nb; e += 256) {
                const int i = e / nb, k = e - (e / nb) * nb;
                P[i * LDP + k] = A[(size_t)(j0 + i) * ld + j0 + k];
            }
            __syncthreads();
            for (int k = 0; k < nb; ++k) {
                const float ex = P[k * LDP + k];
                const float l = sqrtf(1.f + ex);
                __syncthreads();
                if (tid == 0) {
                    P[k * LDP + k] = l;
                    if (INSEG) dR[start + j0 + k] = 0.5f * log1pf(ex);
                }
                for (int i = k + 1 + tid; i < m; i += 256) P[i * LDP + k] = P[i * LDP + k] / l;
                __syncthreads();
                const int w = nb - k - 1;
                if (w > 0) {
                    const int cnt = (m - k - 1) * w;
                    for (int e = tid; e < cnt; e += 256) {
                        const int i = k + 1 + e / w;
                        const int p = k + 1 + (e - (e / w) * w);
                        if (i >= p) P[i * LDP + p] -= P[i * LDP + k] * P[p * LDP + k];
                    }
                }
                __syncthreads();
            }
            for (int e = tid; e < m * nb; e += 256) {
                const int i = e / nb, k = e - (e / nb) * nb;
                if (i >= k) A[(size_t)(j0 + i) * ld + j0 + k] = P[i * LDP + k];
            }
            const int j1 = j0 + nb;
            if (j1 < ncols) {
                const int tr = (nrows - j1 + 63) / 64, tc = (ncols - j1 + 63) / 64;
                const int ty = tid >> 4, tx = tid & 15;
                const int rb = j1 - j0;   // panel row of global row j1
                for (int I = 0; I < tr; ++I) {
                    const int jmax = min(I, tc - 1);
                    for (int J = 0; J <= jmax; ++J) {
                        float acc[4][4] = {};
                        int ra[4], rbv[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            ra[q] = min(rb + I * 64 + ty * 4 + q, m - 1);
                            rbv[q] = min(rb + J * 64 + tx * 4 + q, m - 1);
                        }
                        for (int k = 0; k < nb; ++k) {
                            float a[4], b[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) { a[q] = P[ra[q] * LDP + k]; b[q] = P[rbv[q] * LDP + k]; }
#pragma unroll
                            for (int q = 0; q < 4; ++q)
#pragma unroll
                                for (int r = 0; r < 4; ++r) acc[q][r] = fmaf(a[q], b[r], acc[q][r]);
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int i = j1 + I * 64 + ty * 4 + q;
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const int p = j1 + J * 64 + tx * 4 + r;
                                if (i < nrows && p < ncols && p <= i) A[(size_t)i * ld + p] -= acc[q][r];
                            }
                        }
                    }
                }
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------- in-segment Gram
// G'_s = c Y_s Y_s^T on lower 64 x 64 tiles; grid (seg, 36 tiles).
__global__ void __launch_bounds__(256) ygram_kernel(Segs S, const float *aug, int64_t d, float c,
                                                    float *gp) {
    const int s = blockIdx.x;
    if (s >= *S.nseg || S.k[s] == 0) return;
    const int t = blockIdx.y;
    int I = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
    while ((I + 1) * (I + 2) / 2 <= t) ++I;
    while (I * (I + 1) / 2 > t) --I;
    const int J = t - I * (I + 1) / 2;
    const int len = S.len[s];
    if (I * 64 >= len) return;
    const float *Y = aug + (size_t)s * (size_t)(d + kSegMax) * (size_t)d + (size_t)d * d;
    float *G = gp + (size_t)S.start[s] * kSegMax;
    __shared__ float As[64][33];
    __shared__ float Bs[64][33];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < d; k0 += 32) {
        for (int e = tid; e < 64 * 32; e += 256) {
            const int rr = e >> 5, kk = e & 31;
            const int ia = I * 64 + rr, ib = J * 64 + rr;
            As[rr][kk] = ia < len ? Y[(size_t)ia * d + k0 + kk] : 0.f;
            Bs[rr][kk] = ib < len ? Y[(size_t)ib * d + k0 + kk] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) { a[q] = As[ty * 4 + q][kk]; b[q] = Bs[tx * 4 + q][kk]; }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[q][r] = fmaf(a[q], b[r], acc[q][r]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int i = I * 64 + ty * 4 + q;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int j = J * 64 + tx * 4 + r;
            if (i < len && j < len && j <= i) G[(size_t)i * len + j] = c * acc[q][r];
        }
    }
}

// ---------------------------------------------------------------- first segment
// M = I at a row's start: dR from the float64 Cholesky of I + c X X^T (len <= 64).
template <class IN>
__global__ void __launch_bounds__(256) first_seg_kernel(const IN *__restrict__ H, int64_t d, Segs S,
                                                        double c, float *dR) {
    extern __shared__ double sm1[];
    double *G = sm1;                                   // 64 x 65
    float *X = reinterpret_cast<float *>(sm1 + 64 * 65);  // len x (d + 1), padded rows
    const int64_t ldx = d + 1;
    const int tid = threadIdx.x;
    const int nseg = *S.nseg;
    for (int s = blockIdx.x; s < nseg; s += gridDim.x) {
        if (S.k[s] != 0) continue;
        const int len = S.len[s];
        const int64_t start = S.start[s];
        for (int64_t e = tid; e < (int64_t)len * d; e += 256) X[(e / d) * ldx + (e % d)] = ld_f(H + start * d + e);
        __syncthreads();
        for (int e = tid; e < len * len; e += 256) {
            const int i = e / len, j = e - (e / len) * len;
            if (j <= i) {
                double acc = 0.0;
                for (int k = 0; k < d; ++k) acc += (double)X[i * ldx + k] * (double)X[j * ldx + k];
                G[i * 65 + j] = c * acc;
            }
        }
        __syncthreads();
        for (int k = 0; k < len; ++k) {
            const double ex = G[k * 65 + k];
            const double l = sqrt(1.0 + ex);
            __syncthreads();
            if (tid == 0) dR[start + k] = (float)(0.5 * log1p(ex));
            for (int i = k + 1 + tid; i < len; i += 256) G[i * 65 + k] /= l;
            __syncthreads();
            const int w = len - k - 1;
            for (int e = tid; e < w * w; e += 256) {
                const int i = k + 1 + e / w, p = k + 1 + (e - (e / w) * w);
                if (i >= p) G[i * 65 + p] -= G[i * 65 + k] * G[p * 65 + k];
            }
            __syncthreads();
        }
    }
}

template <int D>
void launch_gram_tc(const __nv_bfloat16 *H, int64_t ns, const Segs &segs, float *mats, size_t mat_stride,
                    int32_t *st, cudaStream_t stream, bool lower = false) {
    using C = GramTC<D>;
    cudaFuncSetAttribute(gram_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    gram_tc_kernel<D><<<dim3((unsigned)ns, (unsigned)C::GROUPS), 256, C::SMEM, stream>>>(H, segs, mats,
                                                                                       mat_stride, lower, st);
}

inline void launch_gram(const float *H, int64_t d, int64_t ns, const Layout &L, int32_t *st,
                        cudaStream_t stream) {
    gram_kernel<float><<<dim3((unsigned)ns, (unsigned)((d / 64) * (d / 64))), 256, 0, stream>>>(
        H, d, L.segs, L.aug, st);
}

inline void launch_gram(const __nv_bfloat16 *H, int64_t d, int64_t ns, const Layout &L, int32_t *st,
                        cudaStream_t stream) {
    const size_t stride = (size_t)(d + kSegMax) * (size_t)d;
    switch (d) {
        case 128: launch_gram_tc<128>(H, ns, L.segs, L.aug, stride, st, stream); return;
        case 256: launch_gram_tc<256>(H, ns, L.segs, L.aug, stride, st, stream); return;
        case 512: launch_gram_tc<512>(H, ns, L.segs, L.aug, stride, st, stream); return;
        default:
            gram_kernel<__nv_bfloat16><<<dim3((unsigned)ns, (unsigned)((d / 64) * (d / 64))), 256, 0, stream>>>(
                H, d, L.segs, L.aug, st);
    }
}

template <class IN>
dbc_status run(const IN *H, const int64_t *offsets, int64_t rows, int64_t T, int64_t N, int64_t d,
               float eps2, float *dR, const Layout &L, int32_t *st, cudaStream_t stream) {
    const double c = (double)d / (double)eps2;
    const int64_t ns = nseg_upper(rows, N);
    const int sms = num_sms();
    seg_table_kernel<<<1, 1024, 0, stream>>>(offsets, rows, T, N, ns, kSegMax, L.segs, st);
    launch_gram(H, d, ns, L, st, stream);
    prefix_kernel<<<dim3((unsigned)rows, (unsigned)((d * d + 255) / 256)), 256, 0, stream>>>(
        L.segs, L.aug, d, c);
    fill_x_kernel<IN><<<dim3((unsigned)ns, 16), 256, 0, stream>>>(H, d, L.segs, L.aug);
    const int chol_grid = (int)std::min<int64_t>(ns, (int64_t)sms * 4);
    const size_t smem_f = (size_t)(d + kSegMax) * (PW + 1) * sizeof(float);
    const size_t smem_i = (size_t)kSegMax * (PW + 1) * sizeof(float);
    cudaFuncSetAttribute(chol_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_f);
    cudaFuncSetAttribute(chol_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_i);
    chol_kernel<false><<<chol_grid, 256, smem_f, stream>>>(L.segs, L.aug, L.gp, d, dR);
    ygram_kernel<<<dim3((unsigned)ns, 36), 256, 0, stream>>>(L.segs, L.aug, d, (float)c, L.gp);
    chol_kernel<true><<<chol_grid, 256, smem_i, stream>>>(L.segs, L.aug, L.gp, d, dR);
    const size_t smem1 = 64 * 65 * sizeof(double) + (size_t)64 * (d + 1) * sizeof(float);
    cudaFuncSetAttribute(first_seg_kernel<IN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    first_seg_kernel<IN><<<(unsigned)std::min<int64_t>(ns, (int64_t)sms * 2), 256, smem1, stream>>>(
        H, d, L.segs, c, dR);
    count_launches(8);
    return launch_status();
}

}  // namespace cr
}  // namespace dbc

#include "segment_tc.cuh"

using namespace dbc;

static bool use_tensor_path(int dtype, int64_t d) {
    return dtype == DBC_BF16 && (d == 128 || d == 256 || d == 512);
}

extern "C" size_t chunk_coding_rate_workspace(int64_t rows, int64_t T, int64_t N, int64_t d) {
    (void)T;
    if (rows < 0 || N < 0 || d <= 0) return 0;
    // large enough for either path (the dtype is not an argument of the query)
    return std::max({cr::carve(nullptr, rows, N, d).bytes, cr::carve2(nullptr, rows, N, d).bytes,
                     cr::carve3(nullptr, rows, N, d).bytes});
}

extern "C" dbc_status chunk_coding_rate(const void *H, int dtype, const int64_t *offsets,
                                        int64_t rows, int64_t T, int64_t N, int64_t d,
                                        float eps2, float *dR, void *ws, size_t ws_bytes,
                                        int32_t *dev_status, dbc_stream_t stream) {
    DBC_NVTX_RANGE("chunk_coding_rate");
    if (rows < 0 || T < 0 || N < 0 || !(eps2 > 0.f) || !isfinite(eps2)) return DBC_ERR_INVALID_ARG;
    if (dtype != DBC_F32 && dtype != DBC_BF16) return DBC_ERR_UNSUPPORTED;
    if (d != 64 && d != 128 && d != 256 && d != 512) return DBC_ERR_UNSUPPORTED;
    if (!offsets && N != rows * T) return DBC_ERR_INVALID_ARG;
    if (N == 0 || rows == 0) return DBC_OK;
    if (!H || !dR || !aligned16(H)) return DBC_ERR_INVALID_ARG;
    if (cr::nseg_upper(rows, N, 256) > INT32_MAX / 2) return DBC_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == DBC_BF16 && d == 256) {
        const cr::Layout3 need3 = cr::carve3(nullptr, rows, N, d);
        if (!ws || ws_bytes < need3.bytes || (reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)))
            return DBC_ERR_WORKSPACE;
        return cr::run_tmem(static_cast<const __nv_bfloat16 *>(H), offsets, rows, T, N, eps2, dR,
                            cr::carve3(ws, rows, N, d), dev_status, s);
    }
    if (use_tensor_path(dtype, d)) {
        const cr::Layout2 need2 = cr::carve2(nullptr, rows, N, d);
        if (!ws || ws_bytes < need2.bytes || (reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)))
            return DBC_ERR_WORKSPACE;
        const cr::Layout2 L2 = cr::carve2(ws, rows, N, d);
        const __nv_bfloat16 *Hb = static_cast<const __nv_bfloat16 *>(H);
        switch (d) {
            case 128: return cr::run_tc<128>(Hb, offsets, rows, T, N, eps2, dR, L2, dev_status, s);
            case 256: return cr::run_tc<256>(Hb, offsets, rows, T, N, eps2, dR, L2, dev_status, s);
            default: return cr::run_tc<512>(Hb, offsets, rows, T, N, eps2, dR, L2, dev_status, s);
        }
    }
    const cr::Layout need = cr::carve(nullptr, rows, N, d);
    if (!ws || ws_bytes < need.bytes || (reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)))
        return DBC_ERR_WORKSPACE;
    const cr::Layout L = cr::carve(ws, rows, N, d);
    if (dtype == DBC_BF16)
        return cr::run(static_cast<const __nv_bfloat16 *>(H), offsets, rows, T, N, d, eps2, dR, L,
                       dev_status, s);
    return cr::run(static_cast<const float *>(H), offsets, rows, T, N, d, eps2, dR, L, dev_status, s);
}

// Streaming continuation: n new positions of each of `streams` streams that have
// already consumed t0 positions (bf16, d = 256).
extern "C" size_t chunk_coding_rate_stream_workspace(int64_t streams, int64_t n, int64_t t0, int64_t d) {
    if (streams < 0 || n < 0 || t0 < 0 || d != 256) return 0;
    int64_t k1 = 0, cnt = 0;
    cr::stream_pieces(t0, n, k1, cnt);
    return cr::carve3(nullptr, streams, streams * n, d, streams * cnt).bytes;
}

extern "C" dbc_status chunk_coding_rate_stream(const void *H, int dtype, int64_t streams, int64_t n, int64_t d,
                                               int64_t t0, float eps2, double *state, float *dR, void *ws,
                                               size_t ws_bytes, int32_t *dev_status, dbc_stream_t stream) {
    DBC_NVTX_RANGE("chunk_coding_rate_stream");
    if (streams < 0 || n < 0 || t0 < 0 || !(eps2 > 0.f) || !isfinite(eps2)) return DBC_ERR_INVALID_ARG;
    if (dtype != DBC_BF16 || d != 256) return DBC_ERR_UNSUPPORTED;
    if (streams == 0 || n == 0) return DBC_OK;
    if (!H || !dR || !state || !aligned16(H) || !aligned16(state)) return DBC_ERR_INVALID_ARG;
    if (streams * n > INT32_MAX || t0 > ((int64_t)1 << 40)) return DBC_ERR_UNSUPPORTED;
    int64_t k1 = 0, cnt = 0;
    cr::stream_pieces(t0, n, k1, cnt);
    if (streams * cnt > INT32_MAX / 2) return DBC_ERR_UNSUPPORTED;
    const cr::Layout3 need = cr::carve3(nullptr, streams, streams * n, d, streams * cnt);
    if (!ws || ws_bytes < need.bytes || (reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)))
        return DBC_ERR_WORKSPACE;
    return cr::run_tmem_stream(static_cast<const __nv_bfloat16 *>(H), streams, n, t0, k1, cnt, eps2, state, dR,
                               cr::carve3(ws, streams, streams * n, d, streams * cnt), dev_status,
                               reinterpret_cast<cudaStream_t>(stream));
}
