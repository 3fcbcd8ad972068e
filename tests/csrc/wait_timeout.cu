// Test kernel for the bounded mbarrier wait of the decode pipeline: it waits on a
// barrier that nothing ever arrives on, through the library's own
// mbar_wait_bounded, so the wait must give up after its cycle limit, raise
// PA_FLAG_TIMEOUT in the caller's flag and return false -- leaving the kernel
// to finish and the context usable.  Test infrastructure only.
#include "../../paged_kv_cache_349_b200/csrc/pa_common.cuh"

namespace {

__global__ void wait_on_silent_barrier(int32_t *flag, int *result, long long *cycles) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        pa::mbar_init(&bar, 1);  // expects one arrival; none ever comes
        pa::fence_mbar_init();
    }
    __syncthreads();
    const long long t0 = clock64();
    // A fresh barrier is in phase 0: waiting for parity 0 waits for an arrival.
    const bool got = pa::mbar_wait_bounded(&bar, 0, flag);
    if (threadIdx.x == 0) {
        *result = got ? 1 : 0;
        *cycles = clock64() - t0;
    }
}

}  // namespace

extern "C" int run_wait_timeout(int32_t *flag, int *result, long long *cycles, long long *limit) {
    *limit = pa::kWaitLimitCycles;
    wait_on_silent_barrier<<<1, 32>>>(flag, result, cycles);
    return cudaGetLastError() == cudaSuccess ? 0 : 1;
}
