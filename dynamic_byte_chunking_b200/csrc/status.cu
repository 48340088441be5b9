// Library-level entry points: status names and version.
#include <atomic>

#include "common.cuh"

static std::atomic<unsigned long long> g_launches{0};

void dbc::count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

extern "C" uint64_t dbc_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

extern "C" const char *dbc_status_string(int status) {
    switch (status) {
        case DBC_OK: return "DBC_OK";
        case DBC_ERR_INVALID_ARG: return "DBC_ERR_INVALID_ARG";
        case DBC_ERR_UNSUPPORTED: return "DBC_ERR_UNSUPPORTED";
        case DBC_ERR_CUDA: return "DBC_ERR_CUDA";
        case DBC_ERR_NONFINITE: return "DBC_ERR_NONFINITE";
        case DBC_ERR_TIMEOUT: return "DBC_ERR_TIMEOUT";
        case DBC_ERR_BOUNDS: return "DBC_ERR_BOUNDS";
        case DBC_ERR_WORKSPACE: return "DBC_ERR_WORKSPACE";
        default: return "DBC_ERR_UNKNOWN";
    }
}

extern "C" int dbc_version(void) { return 100; }
