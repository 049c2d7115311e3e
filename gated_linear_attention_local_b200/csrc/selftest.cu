// Self-test of the bounded mbarrier wait that every pipeline of the tensor-core
// kernels relies on (the pages have no counterpart: it checks this library's own
// failure detection).  One CTA waits on an mbarrier phase that nothing will ever
// complete: thread 0 must give up after the wall-time limit and raise the CTA's abort
// flag, and a thread of another warp waiting on the same phase must then give up
// through that flag.  The kernel records SGLA_DEVICE_TIMEOUT when both returned.
#include "kernels.h"
#include "tc_ptx.cuh"

namespace sgla {

using namespace tc;

__global__ void wait_timeout_selftest_kernel(int *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    __shared__ int gave_up[2];
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none will come
        abort_flag = 0;
        gave_up[0] = gave_up[1] = 0;
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 || threadIdx.x == 32) {
        const bool completed = mbar_wait(&bar, 0, reinterpret_cast<volatile int *>(&abort_flag));
        gave_up[threadIdx.x >> 5] = completed ? 0 : 1;
    }
    __syncthreads();
    if (threadIdx.x == 0) *status = (gave_up[0] && gave_up[1] && abort_flag) ? kDevTimeout : kDevOk;
}

cudaError_t launch_wait_timeout_selftest(int *status, cudaStream_t st) {
    wait_timeout_selftest_kernel<<<1, 64, 0, st>>>(status);
    return cudaGetLastError();
}

}  // namespace sgla
