// chunk_topk_select: boundary positions per row.
//
// ByteFlow (papernotes.org notes, "Key design 2"; paper.rainbus.top summary,
// "Method steps", stage 2): the first position is always a boundary, the K-1
// positions with the largest dR among t >= 1 join it, and the K boundaries are
// listed in time order.  Ties are broken towards the earlier position.
//
// Rows of up to kClusterKeys candidates (all the workloads' rows) are selected
// by a cluster of kCluster CTAs per row, each holding a contiguous slice of the
// row's keys in shared memory: every radix pass builds the slice histograms,
// each CTA reads the others' histograms through distributed shared memory
// (plain loads, no multicast) and takes the same decision, and the ordered
// compaction offsets each slice by the counts of the slices before it.
// Longer rows take one CTA per row: the row's dR values become order-preserving 32-bit keys
// (in shared memory when they fit), a 4-pass 8-bit radix select finds the
// (K-1)-th largest key v and how many keys equal to v are still needed (the
// histogram increments are aggregated per warp: the keys of a row share their
// leading bytes), and one ordered pass writes the selected positions, which are
// then already in increasing order (no sort).
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace dbc {
namespace tk {

constexpr int kThreads = 1024;
constexpr int kSmemKeys = 48 * 1024;   // keys held in shared memory (192 KB)

__device__ __forceinline__ uint32_t key_of(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;                      // -0 and +0 are equal
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide scan of v over kThreads threads; *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int *wsum, int *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int w = wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    const int r = (wid ? wsum[wid - 1] : 0) + x - v;
    *total = wsum[31];
    __syncthreads();
    return r;
}

__device__ __forceinline__ int64_t row_K(const int64_t *Kp, int64_t Ks, int64_t r, int32_t *st) {
    int64_t K = Kp ? Kp[r] : Ks;
    if (K < 1) {
        flag(st, DBC_ERR_BOUNDS);
        K = 1;
    }
    return K;
}

__global__ void __launch_bounds__(1024) offsets_kernel(const int64_t *offsets, int64_t rows, int64_t T,
                                                       const int64_t *Kp, int64_t Ks,
                                                       int64_t *idx_offsets, int32_t *st) {
    __shared__ int64_t wsum[32];
    __shared__ int64_t carry;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int64_t base = 0; base < rows; base += blockDim.x) {
        const int64_t r = base + tid;
        int64_t cnt = 0;
        if (r < rows) {
            int64_t a, n;
            row_bounds(offsets, r, T, a, n);
            const int64_t K = row_K(Kp, Ks, r, st);
            cnt = n < K ? n : K;
        }
        int64_t x = cnt;
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int64_t w = wsum[lane];
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            wsum[lane] = w;
        }
        __syncthreads();
        const int64_t excl = carry + (wid ? wsum[wid - 1] : 0) + x - cnt;
        if (r < rows) idx_offsets[r] = excl;
        __syncthreads();
        if (tid == (int)blockDim.x - 1) carry = excl + cnt;
        __syncthreads();
    }
    if (tid == 0) idx_offsets[rows] = carry;
}

// Histogram increment with a warp-uniform fast path: the keys of a row share
// their leading bytes (positive values of a narrow range), so in the early
// passes all matching lanes of a warp usually fall into one bin, and one lane
// adds their count; otherwise every lane adds its own (shared atomics).
__device__ __forceinline__ void hist_add(uint32_t *hist, bool match, uint32_t bin) {
    const unsigned active = __ballot_sync(0xffffffffu, match);
    if (!active) return;
    const int leader = __ffs(active) - 1;
    const uint32_t b0 = __shfl_sync(0xffffffffu, bin, leader);
    const bool same = __all_sync(0xffffffffu, !match || bin == b0);
    if (same) {
        if ((int)(threadIdx.x & 31) == leader) atomicAdd(&hist[b0], (uint32_t)__popc(active));
    } else if (match) {
        atomicAdd(&hist[bin], 1u);
    }
}

constexpr int kPerThread = 8;                         // consecutive keys per thread in the compaction
constexpr int kTile = kThreads * kPerThread;          // keys per compaction tile

// dense_K > 0: dense rows with one K for all rows, row r's indices start at
// r * min(K, T) and this kernel writes idx_offsets; otherwise idx_offsets was
// written by offsets_kernel.
__global__ void __launch_bounds__(kThreads) select_kernel(const float *__restrict__ dR,
                                                          const int64_t *offsets, int64_t rows, int64_t T,
                                                          const int64_t *Kp, int64_t Ks, int64_t dense_K,
                                                          int64_t *idx_offsets, int64_t *idx,
                                                          int keys_in_smem, int32_t *st) {
    extern __shared__ uint32_t keys[];
    __shared__ uint32_t hist[256];
    __shared__ int wsum[32];
    __shared__ uint32_t s_bin;
    __shared__ int64_t s_rem;
    const int tid = threadIdx.x;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        int64_t a, n;
        row_bounds(offsets, r, T, a, n);
        const int64_t K = row_K(Kp, Ks, r, nullptr);
        int64_t obase;
        if (dense_K > 0) {
            const int64_t per = T < dense_K ? T : dense_K;
            obase = r * per;
            if (tid == 0) {
                idx_offsets[r] = obase;
                if (r == rows - 1) idx_offsets[rows] = rows * per;
            }
        } else {
            obase = idx_offsets[r];
        }
        int64_t *out = idx + obase;
        if (n <= 0) continue;
        if (K >= n) {
            for (int64_t t = tid; t < n; t += kThreads) out[t] = t;
            continue;
        }
        if (tid == 0) out[0] = 0;
        const int64_t need = K - 1;
        if (need == 0) continue;
        const int64_t m = n - 1;                 // candidates are t = 1 .. n-1
        const float *row = dR + a + 1;
        const bool in_smem = m <= keys_in_smem;
        bool bad = false;
        if (in_smem) {
            for (int64_t j = tid; j < m; j += kThreads) {
                const float f = row[j];
                bad |= !isfinite(f);
                keys[j] = key_of(f);
            }
        } else {
            for (int64_t j = tid; j < m; j += kThreads) bad |= !isfinite(row[j]);
        }
        if (bad) flag(st, DBC_ERR_NONFINITE);
        __syncthreads();
        uint32_t prefix = 0, mask = 0;
        int64_t rem = need;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int b = tid; b < 256; b += kThreads) hist[b] = 0;
            __syncthreads();
            for (int64_t base = 0; base < m; base += kThreads) {   // uniform trip count: whole warps
                const int64_t j = base + tid;
                uint32_t k = 0;
                if (j < m) k = in_smem ? keys[j] : key_of(row[j]);
                hist_add(hist, j < m && (k & mask) == prefix, (k >> shift) & 255u);
            }
            __syncthreads();
            if (tid < 32) {
                // warp 0: suffix sums over 8 bins per lane, then pick the bin
                uint32_t c8[8];
                uint32_t loc = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) { c8[q] = hist[255 - (tid * 8 + q)]; loc += c8[q]; }
                uint32_t inc = loc;   // inclusive prefix over lanes (from the top bin down)
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
                    if (tid >= o) inc += y;
                }
                const uint32_t before = inc - loc;
                const bool mine = (int64_t)before < rem && (int64_t)inc >= rem;
                if (mine) {
                    uint32_t cum = before;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if ((int64_t)(cum + c8[q]) >= rem) {
                            s_bin = 255u - (uint32_t)(tid * 8 + q);
                            s_rem = rem - (int64_t)cum;
                            break;
                        }
                        cum += c8[q];
                    }
                }
            }
            __syncthreads();
            prefix |= s_bin << shift;
            mask |= 255u << shift;
            rem = s_rem;
            __syncthreads();
        }
        // ordered compaction: key > v, or key == v among the first `rem` equal keys.  Each thread
        // takes kPerThread consecutive keys of a tile; two block scans per tile place its output.
        const uint32_t v = prefix;
        int64_t carry_eq = 0, carry_sel = 0;
        for (int64_t base = 0; base < m; base += kTile) {
            const int64_t j0 = base + (int64_t)tid * kPerThread;
            uint32_t kk[kPerThread];
            int n_eq = 0, n_gt = 0;
#pragma unroll
            for (int q = 0; q < kPerThread; ++q) {
                const int64_t j = j0 + q;
                kk[q] = 0;
                if (j < m) kk[q] = in_smem ? keys[j] : key_of(row[j]);
                n_eq += (j < m && kk[q] == v) ? 1 : 0;
                n_gt += (j < m && kk[q] > v) ? 1 : 0;
            }
            int tot_eq;
            const int eq_base = block_excl_scan(n_eq, wsum, &tot_eq);
            // equal keys of this thread that are still within the first `rem` of the row
            const int64_t left = rem - (carry_eq + eq_base);
            const int take_eq = left <= 0 ? 0 : (left >= n_eq ? n_eq : (int)left);
            int tot_sel;
            const int sel_base = block_excl_scan(n_gt + take_eq, wsum, &tot_sel);
            int64_t o = 1 + carry_sel + sel_base;
            int eq_seen = 0;
#pragma unroll
            for (int q = 0; q < kPerThread; ++q) {
                const int64_t j = j0 + q;
                if (j < m) {
                    const bool eq = kk[q] == v;
                    if (kk[q] > v || (eq && eq_seen < take_eq)) {
                        if (dcheck(o <= need, st)) out[o] = j + 1;     // slots 1 .. K-1 of the row
                        ++o;
                    }
                    eq_seen += eq ? 1 : 0;
                }
            }
            carry_eq += tot_eq;
            carry_sel += tot_sel;
        }
        __syncthreads();
    }
}


// ---------------------------------------------------------------- cluster per row
constexpr int kCluster = 8;
constexpr int kCThreads = 256;
constexpr int kCWarps = kCThreads / 32;
constexpr int kSliceKeys = 8192;                       // keys per CTA slice (32 KB)
constexpr int kClusterKeys = kCluster * kSliceKeys;    // candidates per row on this path

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kCThreads)
    select_cluster_kernel(const float *__restrict__ dR, const int64_t *offsets, int64_t rows, int64_t T,
                          const int64_t *Kp, int64_t Ks, int64_t dense_K, int64_t *idx_offsets, int64_t *idx,
                          int32_t *st) {
    __shared__ uint32_t keys[kSliceKeys];
    __shared__ uint32_t hist[2][256];                  // alternate passes: a pass never clears what is read
    __shared__ uint32_t tot[256];
    __shared__ uint32_t s_bin;
    __shared__ int s_rem;
    __shared__ int s_cnt[2];                           // this slice's equal-key and selected counts
    __shared__ int s_weq[kCWarps], s_wgt[kCWarps];     // per-warp equal and above counts
    cg::cluster_group cluster = cg::this_cluster();
    const int q = (int)cluster.block_rank();
    const int64_t r = blockIdx.x / kCluster;
    const int tid = threadIdx.x;
    // every decision below is uniform over the cluster (it depends on the row only)
    int64_t a, n;
    row_bounds(offsets, r, T, a, n);
    const int64_t K = row_K(Kp, Ks, r, nullptr);
    int64_t obase;
    if (dense_K > 0) {
        const int64_t per = T < dense_K ? T : dense_K;
        obase = r * per;
        if (q == 0 && tid == 0) {
            idx_offsets[r] = obase;
            if (r == rows - 1) idx_offsets[rows] = rows * per;
        }
    } else {
        obase = idx_offsets[r];
    }
    int64_t *out = idx + obase;
    if (n <= 0) return;
    if (K >= n) {
        for (int64_t t = (int64_t)q * kCThreads + tid; t < n; t += kCluster * kCThreads) out[t] = t;
        return;
    }
    if (q == 0 && tid == 0) out[0] = 0;
    const int need = (int)(K - 1);
    if (need == 0) return;
    const int m = (int)(n - 1);                        // candidates t = 1 .. n-1 (m <= kClusterKeys)
    const int slice = (m + kCluster - 1) / kCluster;
    const int k0 = q * slice, k1 = min(m, k0 + slice); // this CTA's candidates [k0, k1)
    const int mine = max(0, k1 - k0);
    const float *row = dR + a + 1;
    bool bad = false;
#pragma unroll 4
    for (int j = tid; j < mine; j += kCThreads) {     // four loads in flight
        const float f = row[k0 + j];
        bad |= !isfinite(f);
        keys[j] = key_of(f);
    }
    if (bad) flag(st, DBC_ERR_NONFINITE);
    uint32_t prefix = 0, mask = 0;
    int rem = need;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        uint32_t *h = hist[pass & 1];
        h[tid] = 0;                                    // kCThreads == 256 bins
        __syncthreads();
        for (int base = 0; base < mine; base += kCThreads) {     // uniform trip count: whole warps
            const int j = base + tid;
            const uint32_t k = j < mine ? keys[j] : 0u;
            hist_add(h, j < mine && (k & mask) == prefix, (k >> shift) & 255u);
        }
        cluster.sync();                                // every slice's histogram is complete
        uint32_t total = 0;
#pragma unroll
        for (int c = 0; c < kCluster; ++c) total += cluster.map_shared_rank(h, c)[tid];
        tot[tid] = total;
        __syncthreads();
        if (tid < 32) {
            // warp 0: suffix sums over 8 bins per lane (from the top bin down), then pick the bin
            uint32_t c8[8];
            uint32_t loc = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) { c8[b] = tot[255 - (tid * 8 + b)]; loc += c8[b]; }
            uint32_t inc = loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
                if (tid >= o) inc += y;
            }
            const uint32_t before = inc - loc;
            if ((int)before < rem && (int)inc >= rem) {
                uint32_t cum = before;
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    if ((int)(cum + c8[b]) >= rem) {
                        s_bin = 255u - (uint32_t)(tid * 8 + b);
                        s_rem = rem - (int)cum;
                        break;
                    }
                    cum += c8[b];
                }
            }
        }
        __syncthreads();
        prefix |= s_bin << shift;
        mask |= 255u << shift;
        rem = s_rem;
    }
    // ordered compaction: key > v, or key == v among the first `rem` equal keys of the row.  The
    // slice's keys are split into eight contiguous ranges, one per warp, of a multiple of 32 keys;
    // warp w walks its range 32 at a time (lane l takes key step * 32 + l: conflict-free shared
    // loads), ranking with ballots; warps are offset by the warps before them, slices by the slices
    // before them.
    const uint32_t v = prefix;
    const int lane = tid & 31, wid = tid >> 5;
    const unsigned lt = (1u << lane) - 1u;
    const int wkeys = ((mine + kCWarps * 32 - 1) / (kCWarps * 32)) * 32;   // keys per warp
    const int wk0 = wid * wkeys;
    const int wsteps = wkeys / 32;
    int n_eq = 0, n_gt = 0;                            // warp totals (every lane holds them)
    for (int step = 0; step < wsteps; ++step) {
        const int j = wk0 + step * 32 + lane;
        const uint32_t k = j < mine ? keys[j] : 0u;
        n_eq += __popc(__ballot_sync(0xffffffffu, j < mine && k == v));
        n_gt += __popc(__ballot_sync(0xffffffffu, j < mine && k > v));
    }
    if (lane == 0) {
        s_weq[wid] = n_eq;
        s_wgt[wid] = n_gt;
    }
    __syncthreads();
    if (tid == 0) {
        int e = 0, g = 0;
        for (int w = 0; w < kCWarps; ++w) { e += s_weq[w]; g += s_wgt[w]; }
        s_cnt[0] = e;                                  // equal keys of the slice
        s_cnt[1] = g;                                  // keys above v in the slice
    }
    cluster.sync();
    // One exchange gives every offset: slice c takes min(eq_c, rem - (equal keys before it)) of its
    // equal keys, so the selected keys before this warp follow from the (equal, above) counts of
    // the slices and warps before it.
    int eq_before = 0, sel_before = 0;
    for (int c = 0; c < q; ++c) {
        const int *rc = cluster.map_shared_rank(s_cnt, c);
        const int e = rc[0], g = rc[1];
        const int l = rem - eq_before;
        sel_before += g + (l <= 0 ? 0 : (l >= e ? e : l));
        eq_before += e;
    }
    // this CTA's reads of the other slices' counts are done; its own may still be read
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    for (int w = 0; w < wid; ++w) {
        const int e = s_weq[w], g = s_wgt[w];
        const int l = rem - eq_before;
        sel_before += g + (l <= 0 ? 0 : (l >= e ? e : l));
        eq_before += e;
    }
    const int left = rem - eq_before;
    const int take_eq = left <= 0 ? 0 : (left >= n_eq ? n_eq : left);
    int64_t o = 1 + (int64_t)sel_before;
    int eq_run = 0;
    for (int step = 0; step < wsteps; ++step) {
        const int j = wk0 + step * 32 + lane;
        const uint32_t k = j < mine ? keys[j] : 0u;
        const bool eq = j < mine && k == v;
        const unsigned em = __ballot_sync(0xffffffffu, eq);
        const bool sel = (j < mine && k > v) || (eq && eq_run + __popc(em & lt) < take_eq);
        const unsigned sm = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const int64_t at = o + __popc(sm & lt);
            if (dcheck(at <= need, st)) out[at] = k0 + j + 1;
        }
        o += __popc(sm);
        eq_run += __popc(em);
    }
    // no CTA leaves while its counts may still be read
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace tk
}  // namespace dbc

using namespace dbc;

extern "C" size_t chunk_topk_select_workspace(int64_t rows) {
    (void)rows;
    return 0;
}

extern "C" dbc_status chunk_topk_select(const float *dR, const int64_t *offsets, int64_t rows,
                                        int64_t T, int64_t N, const int64_t *K_per_row,
                                        int64_t K_scalar, int64_t *idx, int64_t *idx_offsets,
                                        void *ws, size_t ws_bytes, int32_t *dev_status,
                                        dbc_stream_t stream) {
    DBC_NVTX_RANGE("chunk_topk_select");
    (void)ws; (void)ws_bytes;
    if (rows < 0 || T < 0 || N < 0) return DBC_ERR_INVALID_ARG;
    if (!K_per_row && K_scalar < 1) return DBC_ERR_INVALID_ARG;
    if (!offsets && N != rows * T) return DBC_ERR_INVALID_ARG;
    if (!idx_offsets) return DBC_ERR_INVALID_ARG;
    if (rows > 0 && N > 0 && (!dR || !idx)) return DBC_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // dense rows with one K: the select kernel writes the offsets itself (r * min(K, T))
    const int64_t dense_K = (!offsets && !K_per_row) ? K_scalar : 0;
    if (!dense_K || rows == 0 || N == 0) {
        tk::offsets_kernel<<<1, 1024, 0, s>>>(offsets, rows, T, K_per_row, K_scalar, idx_offsets, dev_status);
        count_launches(1);
    }
    if (rows == 0 || N == 0) return launch_status();
    const int64_t m = T > 1 ? T - 1 : 1;
    if (m <= tk::kClusterKeys && rows <= INT32_MAX / tk::kCluster) {
        // every row fits the cluster path (T is the longest row)
        tk::select_cluster_kernel<<<(unsigned)(rows * tk::kCluster), tk::kCThreads, 0, s>>>(
            dR, offsets, rows, T, K_per_row, K_scalar, dense_K, idx_offsets, idx, dev_status);
        count_launches(1);
        return launch_status();
    }
    const int keys = (int)std::min<int64_t>(m, tk::kSmemKeys);
    const size_t smem = (size_t)keys * sizeof(uint32_t);
    cudaFuncSetAttribute(tk::select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int grid = (int)std::min<int64_t>(rows, 65535);
    tk::select_kernel<<<grid, tk::kThreads, smem, s>>>(dR, offsets, rows, T, K_per_row, K_scalar, dense_K,
                                                       idx_offsets, idx, keys, dev_status);
    count_launches(1);
    return launch_status();
}
