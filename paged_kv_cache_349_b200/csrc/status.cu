// Status strings, version, launch counter and small device queries.
#include <atomic>
#include <mutex>

#include "pa_common.cuh"

namespace pa {

static std::atomic<uint64_t> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int device_sm_count() {
    static std::mutex mu;
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

}  // namespace pa

extern "C" {

const char *pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_BAD_INDEX: return "PA_ERR_BAD_INDEX";
        case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT";
        case PA_ERR_OOM: return "PA_ERR_OOM";
        case PA_ERR_STATE: return "PA_ERR_STATE";
        default: return "PA_ERR_UNKNOWN";
    }
}

int pa_version(void) { return 100; }

uint64_t pa_launch_count(void) { return pa::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
