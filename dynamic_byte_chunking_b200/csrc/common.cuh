// Shared helpers of the dbc kernels: argument checks, workspace carving,
// device status flags, element loads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>

#include "dbc.h"

namespace dbc {

constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t x, size_t a = kWsAlign) { return (x + a - 1) / a * a; }

// Carves 256-byte aligned sub-buffers out of a caller workspace.  With
// base == nullptr it only measures.
struct Carver {
    char *base;
    size_t off = 0;
    explicit Carver(void *b) : base(static_cast<char *>(b)) {}
    template <class T>
    T *take(size_t count) {
        size_t o = off;
        off = align_up(off + count * sizeof(T));
        return base ? reinterpret_cast<T *>(base + o) : nullptr;
    }
};

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline dbc_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DBC_OK : DBC_ERR_CUDA;
}

__device__ __forceinline__ void flag(int32_t *st, int code) {
    if (st) atomicOr(st, 1 << code);
}

// Internal invariants checked on the device in the debug build (compiled with
// -DDBC_DEBUG, libdbc_debug.so): a violated invariant flags DBC_ERR_BOUNDS and
// the caller skips the access instead of trapping.  The release build
// compiles the check away (it always passes).
#ifdef DBC_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool dcheck(bool cond, int32_t *st) {
    if (kDebugChecks && !cond) {
        flag(st, DBC_ERR_BOUNDS);
        return false;
    }
    return true;
}

__device__ __forceinline__ float ld_f(const float *p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// Row bounds of a packed batch: dense when offsets == nullptr.
__device__ __forceinline__ void row_bounds(const int64_t *offsets, int64_t r, int64_t T,
                                           int64_t &a, int64_t &n) {
    if (offsets) {
        a = offsets[r];
        n = offsets[r + 1] - a;
    } else {
        a = r * T;
        n = T;
    }
}

// Index r with idx_offsets[r] <= k < idx_offsets[r+1] (offsets non-decreasing).
__device__ __forceinline__ int64_t find_row(const int64_t *offs, int64_t rows, int64_t k) {
    int64_t lo = 0, hi = rows;  // invariant offs[lo] <= k < offs[hi]
    while (hi - lo > 1) {
        int64_t mid = (lo + hi) >> 1;
        if (offs[mid] <= k) lo = mid; else hi = mid;
    }
    return lo;
}

// Names one C-ABI call in profiler timelines (an NVTX range; header-only, and
// without an attached tool each push/pop is a call through a null hook).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
#define DBC_NVTX_RANGE(name) ::dbc::NvtxRange dbc_nvtx_range_(name)

// Number of kernels the library has launched (all entry points, all threads).
void count_launches(int n);

inline int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
    }
    return n;
}

}  // namespace dbc
