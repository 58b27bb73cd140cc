// selftest.cu -- exercises the bounded-wait path every kernel relies on.
//
// One CTA initialises an mbarrier that nothing ever arrives at and waits on it
// with the same bounded wait (mbar_wait) the decode, prefill and projection
// kernels use.  The wait gives up after `limit_ns` of global time, the kernel
// sets the TIMEOUT status bit and returns normally: no trap, no fault, and the
// context stays usable.  gqa_get_status then reports GQA_ERR_TIMEOUT.
#include "common.cuh"
#include "gqa.h"
#include "internal.h"

namespace gqa {

namespace {

__global__ void wait_timeout_kernel(unsigned *status, unsigned long long limit_ns, int *waited) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = mbar_wait(&bar, 0, limit_ns);  // phase 0 never completes
        if (!ok) set_status(status, STATUS_TIMEOUT);
        if (waited) *waited = ok ? 0 : 1;
    }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned *status, uint64_t limit_ns, int *waited, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(status, limit_ns, waited);
    return cudaGetLastError();
}

}  // namespace gqa
