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
// upper triangle of B in shared memory (158 KB at d = 256, layout below) for
// all the call's positions, moving it in and out as one bulk copy per row;
// thread k owns column k for w and row k for the update.
#include "common.cuh"
#include "tc.cuh"

namespace dbc {
namespace ss {

constexpr int kThreads = 256;      // = the largest d
constexpr int kMaxD = 256;
constexpr int kSkew = 28;          // spare floats per row: a 16-byte-step shift of up to 7 pieces

// Shared layout of the carried factor: row i holds columns (i & ~3) .. d-1 (len(i) = d - (i & ~3)
// floats, a whole number of 16-byte pieces, so each row moves as one bulk copy; the up to three
// entries left of the diagonal are carried along untouched).  Rows are laid out back to back with
// kSkew spare floats each (row_base), and row i starts some whole pieces into its room, chosen so
// that its update thread (thread i: lane i % 32, with the neighbouring rows of similar length in
// the same warp) meets a bank no other lane of its warp meets: at every step the 32 lanes' entries
// (row i, column i + step) fall in 32 different banks.
__device__ __forceinline__ int row_len(int i, int d) { return d - (i & ~3); }
__device__ __forceinline__ int row_base(int i, int d) {
    const int q = i >> 2, r = i & 3;
    return i * (d + kSkew) - 4 * (2 * q * (q - 1) + r * q);
}
__device__ __forceinline__ int row_start(int i, int d) {
    const int b = row_base(i, d);
    return b + 4 * ((((i >> 2) & 7) - (b >> 2)) & 7);
}

inline size_t smem_bytes(int d) {
    const int q = d >> 2;
    return (size_t)(d * (d + kSkew) - 8 * q * (q - 1)) * sizeof(float);
}

template <class IN>
__global__ void __launch_bounds__(kThreads) step_kernel(const IN *__restrict__ H, int64_t n, int d, float sqrt_c,
                                                        float *__restrict__ Bstate, float *__restrict__ dR,
                                                        int32_t *st) {
    extern __shared__ __align__(16) float Bp[];
    // per column k of this position: (w_k, sqrt(beta_{k-1}/beta_k), beta_{k-1}/beta_k, w_k/beta_k)
    __shared__ float4 s_col[kMaxD];
    __shared__ __align__(16) float s_h[kMaxD];
    __shared__ __align__(16) int s_off[kMaxD];       // s_off[i] + c = entry (i, c) for c >= (i & ~3)
    __shared__ float s_wsum[kThreads / 32];
    __shared__ uint64_t mbar;
    const int k = threadIdx.x, lane = k & 31, warp = k >> 5;
    const int64_t s = blockIdx.x;
    float *B = Bstate + s * (int64_t)d * d;
    if (k < d) s_off[k] = row_start(k, d) - (k & ~3);
    if (k == 0) {
        tc::mbar_init(&mbar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    // the carried factor: one bulk copy per row (16-byte aligned on both sides), all in flight at once
    if (k == 0) {
        uint32_t bytes = 0;
        for (int i = 0; i < d; ++i) bytes += 4u * (uint32_t)row_len(i, d);
        tc::mbar_arrive_expect_tx(&mbar, bytes);
    }
    __syncthreads();
    if (k < d)
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                         tc::smem_u32(Bp + row_start(k, d))),
                     "l"(B + (int64_t)k * d + (k & ~3)), "r"(4u * (uint32_t)row_len(k, d)), "r"(tc::smem_u32(&mbar))
                     : "memory");
    bool ok = tc::mbar_wait(&mbar, 0, st);
    if (!ok) ok = tc::mbar_wait(&mbar, 0, st);        // the copies land before the CTA may leave
    ok = __syncthreads_and(ok) != 0;
    if (!ok) return;
    const IN *Hs = H + s * n * (int64_t)d;
    float h_next = k < d && n > 0 ? ld_f(Hs + k) : 0.f;
    for (int64_t t = 0; t < n; ++t) {
        const float hk = h_next;
        if (k < d && !isfinite(hk)) flag(st, DBC_ERR_NONFINITE);
        if (k < d) s_h[k] = hk;
        if (k < d && t + 1 < n) h_next = ld_f(Hs + (t + 1) * d + k);
        __syncthreads();                              // h in place; the last update complete
        // w_k = sqrt(c) sum_{i <= k} B_ik h_i: column k, four rows per round (their offsets and h
        // values as broadcast 16-byte loads), two rounds of loads before the multiply-adds
        float wk = 0.f;
        if (k < d) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            int i = 0;
            for (; i + 8 <= k + 1; i += 8) {
                const int4 o0 = *reinterpret_cast<const int4 *>(s_off + i);
                const int4 o1 = *reinterpret_cast<const int4 *>(s_off + i + 4);
                const float4 h0 = *reinterpret_cast<const float4 *>(s_h + i);
                const float4 h1 = *reinterpret_cast<const float4 *>(s_h + i + 4);
                const float b0 = Bp[o0.x + k], b1 = Bp[o0.y + k], b2 = Bp[o0.z + k], b3 = Bp[o0.w + k];
                const float b4 = Bp[o1.x + k], b5 = Bp[o1.y + k], b6 = Bp[o1.z + k], b7 = Bp[o1.w + k];
                acc[0] = fmaf(b0, h0.x, acc[0]); acc[1] = fmaf(b1, h0.y, acc[1]);
                acc[2] = fmaf(b2, h0.z, acc[2]); acc[3] = fmaf(b3, h0.w, acc[3]);
                acc[4] = fmaf(b4, h1.x, acc[4]); acc[5] = fmaf(b5, h1.y, acc[5]);
                acc[6] = fmaf(b6, h1.z, acc[6]); acc[7] = fmaf(b7, h1.w, acc[7]);
            }
            for (; i <= k; ++i) acc[0] = fmaf(Bp[s_off[i] + k], s_h[i], acc[0]);
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
        // row my_row of B: x solves V x = b (b_j = 0 left of the diagonal, so the sum starts at the
        // diagonal).  Four columns per group, the next group's loads before this group's stores.
        if (k < d) {
            const int r0 = k;
            float *row = Bp + s_off[r0];              // row[j] = B_(r0)j for j >= r0
            float sigma = 0.f;
            const int ng = (d - r0) / 4;
            float b[4], bn[4];
            float4 cl[4], cn[4];
            int j = r0;
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
    // back to the caller's rows, one bulk copy per row (the entries left of the diagonal that a row's
    // first piece carries go back unchanged)
    tc::fence_async_smem();
    __syncthreads();
    if (k < d) {
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(B + (int64_t)k * d + (k & ~3)),
                     "r"(tc::smem_u32(Bp + row_start(k, d))), "r"(4u * (uint32_t)row_len(k, d))
                     : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
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
