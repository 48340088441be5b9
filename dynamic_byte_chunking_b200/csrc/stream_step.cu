// chunk_coding_rate_step: the marginal coding rate of streams, one new
// position at a time, from a carried inverse Cholesky factor.
//
// ByteFlow (paper.rainbus.top summary, "Prerequisites: lossy coding rate" and
// "Method steps", stage 2; its "Limitations and improvements", first point:
// inference sees the sequence through a window; and "Weaknesses of the
// independent analysis": an incremental rank-one update per byte).  With
// M_t = I + c sum_{i<=t} h_i h_i^T = L L^T and B = L^{-T} (upper triangular):
//
//   w   = sqrt(c) B^T h_t            so  |w|^2 = c h_t^T M_{t-1}^{-1} h_t,
//   dR_t = 1/2 log(1 + |w|^2),
//   M_t = L (I + w w^T) L^T = (L V)(L V)^T  with  I + w w^T = V V^T,
//   B'  = B V^{-T}.
//
// The Cholesky factor of identity plus a rank-one term is explicit: with
// beta_k = 1 + sum_{j<=k} w_j^2 (beta_{-1} = 1), V_kk = sqrt(beta_k/beta_{k-1})
// and V_kj = w_k w_j / sqrt(beta_{j-1} beta_j) for k > j.  Each row b of B
// solves V x = b^T by a running sum sigma_k = sum_{j<=k} V_.. terms:
//
//   x_k     = (b_k - w_k sigma_{k-1}) sqrt(beta_{k-1}/beta_k),
//   sigma_k = (beta_{k-1}/beta_k) sigma_{k-1} + (w_k/beta_k) b_k,
//
// so the update of the whole factor is O(d^2) per position with one fused
// multiply-add on each row's serial chain.  One CTA per stream keeps the
// upper triangle of B in shared memory (d(d+1)/2 floats, 129 KB at d = 256)
// for all the call's positions; thread k owns column k for w and row k for
// the update.
#include "common.cuh"

namespace dbc {
namespace ss {

constexpr int kThreads = 256;      // = the largest d
constexpr int kMaxD = 256;

// Offset of row i of the packed upper triangle (row i holds columns i .. d-1).
__device__ __forceinline__ int row_start(int i, int d) { return i * d - (i * (i - 1)) / 2; }

inline size_t smem_bytes(int d) { return (size_t)d * (d + 1) / 2 * sizeof(float); }

template <class IN>
__global__ void __launch_bounds__(kThreads) step_kernel(const IN *__restrict__ H, int64_t n, int d, float sqrt_c,
                                                        float *__restrict__ Bstate, float *__restrict__ dR,
                                                        int32_t *st) {
    extern __shared__ float Bp[];                    // packed upper triangle of B
    // per column k of this position: (w_k, sqrt(beta_{k-1}/beta_k), beta_{k-1}/beta_k, w_k/beta_k)
    __shared__ float4 s_col[kMaxD];
    __shared__ float s_h[kMaxD];
    __shared__ float s_wsum[kThreads / 32];
    const int k = threadIdx.x, lane = k & 31, warp = k >> 5;
    const int64_t s = blockIdx.x;
    float *B = Bstate + s * (int64_t)d * d;
    // the carried factor's upper triangle: row i's entries i .. d-1 are contiguous in both layouts, so
    // every element is one 4-byte asynchronous copy, all in flight at once (16-byte pieces through
    // registers measured no faster)
    {
        const uint32_t sb = (uint32_t)__cvta_generic_to_shared(Bp);
        int o = k;
#pragma unroll 8
        for (int i = 0; i < d; ++i) {
            if (k >= i && k < d)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sb + 4u * (uint32_t)o),
                             "l"(B + (int64_t)i * d + k) : "memory");
            o += d - 1 - i;
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    const IN *Hs = H + s * n * (int64_t)d;
    float h_next = k < d && n > 0 ? ld_f(Hs + k) : 0.f;
    for (int64_t t = 0; t < n; ++t) {
        const float hk = h_next;
        if (k < d && !isfinite(hk)) flag(st, DBC_ERR_NONFINITE);
        if (k < d) s_h[k] = hk;
        if (k < d && t + 1 < n) h_next = ld_f(Hs + (t + 1) * d + k);
        __syncthreads();                              // h in place; the factor (or the last update) complete
        // w_k = sqrt(c) sum_{i <= k} B_ik h_i: column k of the packed rows (row i starts at
        // row_start(i), so the entry moves by d - 1 - i from row i to row i + 1)
        float wk = 0.f;
        if (k < d) {
            // eight rows per round, every load issued before the multiply-adds
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            int i = 0, off = k;                       // off = row_start(i) + (k - i)
            for (; i + 8 <= k + 1; i += 8) {
                float bv[8];
                int o = off;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    bv[u] = Bp[o];
                    o += d - 1 - (i + u);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) acc[u] = fmaf(bv[u], s_h[i + u], acc[u]);
                off = o;
            }
            for (; i <= k; ++i) {
                acc[0] = fmaf(Bp[off], s_h[i], acc[0]);
                off += d - 1 - i;
            }
            wk = ((acc[0] + acc[1]) + (acc[2] + acc[3]) + ((acc[4] + acc[5]) + (acc[6] + acc[7]))) * sqrt_c;
        }
        // inclusive scan of w_k^2 over k: q_k = sum_{j <= k} w_j^2
        const float wk2 = wk * wk;
        float q = wk2;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, q, o);
            if (lane >= o) q += y;
        }
        if (lane == 31) s_wsum[warp] = q;
        __syncthreads();
        float before = 0.f, total = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            const float x = s_wsum[w];
            before += w < warp ? x : 0.f;
            total += x;
        }
        q += before;
        if (k < d) {
            const float beta = 1.f + q, beta_prev = 1.f + (q - wk2);
            const float a = beta_prev / beta;
            s_col[k] = make_float4(wk, sqrtf(a), a, wk / beta);
        }
        if (k == 0) dR[s * n + t] = 0.5f * log1pf(total);
        __syncthreads();
        // row k of B: x solves V x = b (b_j = 0 left of the diagonal, so the sum starts at k).  Four
        // columns per group, the next group's loads before this group's stores (the entries differ).
        // Lanes walk their own rows from their own diagonals: the rows' starts fall in different banks
        // (a warp-aligned walk, with broadcast coefficients, measured slower)
        if (k < d) {
            float *row = Bp + row_start(k, d) - k;    // row[j] = B_kj for j >= k
            float sigma = 0.f;
            const int ng = (d - k) / 4;               // whole groups of four columns
            float b[4], bn[4];
            float4 cl[4], cn[4];
            int j = k;
            if (ng > 0) {
#pragma unroll
                for (int u = 0; u < 4; ++u) { b[u] = row[j + u]; cl[u] = s_col[j + u]; }
            }
            for (int g = 0; g < ng; ++g, j += 4) {
                if (g + 1 < ng) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) { bn[u] = row[j + 4 + u]; cn[u] = s_col[j + 4 + u]; }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float x = (b[u] - cl[u].x * sigma) * cl[u].y;
                    sigma = fmaf(cl[u].z, sigma, cl[u].w * b[u]);
                    b[u] = x;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) row[j + u] = b[u];
#pragma unroll
                for (int u = 0; u < 4; ++u) { b[u] = bn[u]; cl[u] = cn[u]; }
            }
            for (; j < d; ++j) {
                const float bj = row[j];
                const float4 c1 = s_col[j];
                const float x = (bj - c1.x * sigma) * c1.y;
                sigma = fmaf(c1.z, sigma, c1.w * bj);
                row[j] = x;
            }
        }
    }
    __syncthreads();
    // back to the caller's rows, eight rows per round with their shared loads first (the strictly
    // lower triangle is not written)
    {
        int o = k;
        for (int i0 = 0; i0 < d; i0 += 8) {
            float v[8];
            int oo = o;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u;
                v[u] = (i < d && k >= i && k < d) ? Bp[oo] : 0.f;
                oo += d - 1 - i;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u;
                if (i < d && k >= i && k < d) B[(int64_t)i * d + k] = v[u];
            }
            o = oo;
        }
    }
}

}  // namespace ss
}  // namespace dbc

using namespace dbc;

extern "C" dbc_status chunk_coding_rate_step(const void *H, int dtype, int64_t streams, int64_t n, int64_t d,
                                             float eps2, float *B_state, float *dR, int32_t *dev_status,
                                             dbc_stream_t stream) {
    DBC_NVTX_RANGE("chunk_coding_rate_step");
    if (streams < 0 || n < 0 || d <= 0 || !(eps2 > 0.f)) return DBC_ERR_INVALID_ARG;
    if (dtype != DBC_F32 && dtype != DBC_BF16) return DBC_ERR_UNSUPPORTED;
    if (d > ss::kMaxD || d % 4) return DBC_ERR_UNSUPPORTED;
    if (streams == 0 || n == 0) return DBC_OK;
    if (streams > INT32_MAX || !H || !B_state || !dR || !aligned16(B_state)) return DBC_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t smem = ss::smem_bytes((int)d);
    const float sqrt_c = sqrtf((float)d / eps2);
    if (dtype == DBC_BF16) {
        cudaFuncSetAttribute(ss::step_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        ss::step_kernel<__nv_bfloat16><<<(unsigned)streams, ss::kThreads, smem, s>>>(
            static_cast<const __nv_bfloat16 *>(H), n, (int)d, sqrt_c, B_state, dR, dev_status);
    } else {
        cudaFuncSetAttribute(ss::step_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        ss::step_kernel<float><<<(unsigned)streams, ss::kThreads, smem, s>>>(static_cast<const float *>(H), n,
                                                                             (int)d, sqrt_c, B_state, dR,
                                                                             dev_status);
    }
    count_launches(1);
    return launch_status();
}
