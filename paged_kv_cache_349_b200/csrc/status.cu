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

int device_address(const void *p, void **dev_ptr) {
    *dev_ptr = nullptr;
    if (!p) return PA_ERR_INVALID_ARG;
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // clear the (non-sticky) error so the next launch check does not report it
        return PA_ERR_INVALID_ARG;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    switch (a.type) {
    case cudaMemoryTypeDevice:
        if (a.device != dev) return PA_ERR_INVALID_ARG;  // another GPU's memory: not this library's to reach
        *dev_ptr = const_cast<void *>(p);
        return PA_OK;
    case cudaMemoryTypeManaged:
        *dev_ptr = const_cast<void *>(p);
        return PA_OK;
    case cudaMemoryTypeHost:
        if (!a.devicePointer) return PA_ERR_INVALID_ARG;
        // the mapping of the allocation's base, offset to p
        *dev_ptr = static_cast<char *>(a.devicePointer) +
                   (static_cast<const char *>(p) - static_cast<const char *>(a.hostPointer));
        return PA_OK;
    default:
        return PA_ERR_INVALID_ARG;
    }
}

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
