// k_selftest.cu -- self-test of the bounded waits.
//
// Every pipeline of this library waits on mbarriers through mbar_wait
// (common.cuh), which gives up after a time limit, records QSA_DEV_TIMEOUT in
// the status word and lets the kernel return instead of hanging the GPU.  This
// kernel exercises that exit path on purpose, with no fault and no hang: one
// CTA takes TMEM columns as the tensor-core kernels do, waits on an mbarrier
// that nothing ever arrives on, gives up after the caller's limit, releases the
// TMEM and returns.
#include "internal.h"

namespace qsa {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint64_t limit_ns, unsigned *status,
                                                          unsigned *result) {
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);      // expects one arrival; none ever comes
        fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(&tmem_base, 32);
    tmem_relinquish();
    tc_fence_before();
    __syncwarp();
    tc_fence_after();
    bool ok = true;
    if (threadIdx.x == 0) {
        ok = mbar_wait(&bar, 0, status, limit_ns);
        result[0] = ok ? 1u : 0u;   // 0: the wait gave up, as it must
    }
    __syncwarp();
    tc_fence_before();
    tmem_dealloc(tmem_base, 32);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, unsigned *status, unsigned *result, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(limit_ns, status, result);
    return cudaGetLastError();
}

}  // namespace qsa
