// Diagnostic of the device-side failure detection: every pipeline wait of the
// grouped GEMM is an mbarrier wait bounded in global time (ptx::mbar_wait);
// when it gives up, the kernel records MOE_ERR_DEVICE_TIMEOUT in the caller's
// status word and winds down instead of hanging.  This kernel runs that same
// wait on a barrier nothing ever arrives on, so the give-up path can be
// exercised without faulting or hanging a GPU.
#include "common.cuh"
#include "nvtx_range.cuh"
#include "ptx.cuh"

namespace moe {

__global__ void bounded_wait_probe_kernel(int32_t* status, uint64_t limit_ns, uint64_t* elapsed) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = ptx::globaltimer();
        // phase 0 of a fresh barrier with one expected arrival that never comes
        const bool done = ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns);
        if (!done) flag_status(status, MOE_ERR_DEVICE_TIMEOUT);
        if (elapsed) *elapsed = ptx::globaltimer() - t0;
    }
}

}  // namespace moe

extern "C" int moe_selftest_bounded_wait(int32_t* device_status, uint64_t limit_ns,
                                         uint64_t* device_elapsed_ns, void* stream) {
    MOE_NVTX_RANGE();
    using namespace moe;
    if (!device_status || limit_ns < 1000ull || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
    bounded_wait_probe_kernel<<<1, 32, 0, as_stream(stream)>>>(device_status, limit_ns,
                                                               device_elapsed_ns);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
