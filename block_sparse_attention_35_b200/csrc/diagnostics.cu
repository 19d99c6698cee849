// diagnostics.cu - a kernel that exercises the library's bounded wait on a barrier that
// nothing completes, so the timeout path can be tested without hanging a GPU.
#include "pbsa_device.cuh"
#include "pbsa_internal.cuh"

namespace pbsa {

namespace {

__global__ void wait_selftest_kernel(int32_t* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 never completes: the wait must give up and record PBSA_ERR_TIMEOUT
        mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_wait_selftest(int32_t* status, long long timeout_ns, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(status, static_cast<unsigned long long>(timeout_ns));
    return cudaGetLastError();
}

}  // namespace pbsa
