// selftest.cu -- failure-detection self-test of the bounded waits.
//
// One thread waits, through the same bounded_wait every pipeline of the
// library uses, for an mbarrier phase that nothing completes.  The wait
// gives up after its time bound, sets the timeout bit in the device error
// word and the kernel returns: the failure is reported and the context stays
// usable, which is what a broken pipeline does in the real kernels (there
// the other roles also see the shared abort flag, drain their copies and
// free tensor memory before returning).
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

__global__ void wait_timeout_kernel(uint32_t *err)
{
    __shared__ uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort_flag = 0u;
        ptx::fence_barrier_init();
        // Phase 0 completes on one arrival; none comes.
        bounded_wait(&bar, 0u, &abort_flag, err, kErrTimeoutMma);
    }
}

}  // namespace

cudaError_t launch_wait_timeout(uint32_t *err, cudaStream_t s)
{
    wait_timeout_kernel<<<1, 32, 0, s>>>(err);
    return cudaGetLastError();
}

}  // namespace moe
