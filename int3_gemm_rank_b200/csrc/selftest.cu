// selftest.cu -- a self-test of the bounded waits of the sm_100a kernels.
//
// Every wait of the library's kernels on an mbarrier (milo_device.cuh:
// mbar_wait / warp_wait) gives up after a fixed number of SM cycles, flags
// MILO_DEV_TIMEOUT in the caller's status word and lets the CTA unwind, so a
// lost arrival ends as an error the host reads instead of a hung GPU.  This
// entry point runs that wait on a barrier that nothing ever completes.
#include <cuda_runtime.h>

#include "milo_device.cuh"
#include "milo_host.h"

namespace milo {
namespace {

__global__ void wait_selftest_kernel(int32_t* dev_status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    // phase 0 of a fresh barrier completes only when one arrival lands: none does
    if (!warp_wait(&bar, 0) && threadIdx.x == 0) flag(dev_status, MILO_DEV_TIMEOUT);
}

}  // namespace
}  // namespace milo

using namespace milo;

extern "C" milo_status milo_selftest_wait_timeout(int32_t* dev_status, void* stream) {
    clear_error();
    if (!dev_status) return fail(MILO_ERR_INVALID_ARG, "milo_selftest_wait_timeout: NULL dev_status");
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status);
    return check_launch("milo_selftest_wait_timeout");
}
