// ssd_selftest.cu -- a self-test of the library's bounded device waits.
//
// Every mbarrier wait in the tensor-core kernels gives up after a bounded
// number of cycles, records the timeout in a device status word and lets the
// kernel return, so that a lost arrival can never hang the GPU.  The kernel
// here runs that same wait (ptx::mbar_wait) on a barrier that nothing ever
// arrives at, with a short limit: the wait runs out, the status word says so,
// and the host reports SSD_ERR_TIMEOUT.  It exercises the whole timeout path
// without any fault, trap or hang.
#include <cuda_runtime.h>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_prof.h"

#include "tc_ptx.cuh"

namespace ssd {
namespace {

__global__ void k_selftest_wait(long long limit_cycles, int32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // one arrival is expected and none comes: phase 0 never completes
        const bool done = ptx::mbar_wait(&bar, 0, limit_cycles);
        *status = done ? kStatusOk : kStatusTimeout;
    }
}

}  // namespace

void launch_selftest_wait(long long limit_cycles, int32_t* status, cudaStream_t st) {
    ProfScope ps(K_SELFTEST_WAIT, st);
    k_selftest_wait<<<1, 32, 0, st>>>(limit_cycles, status);
}

}  // namespace ssd
