// selftest.cu — exercises the bounded mbarrier wait the kernels use, on a
// barrier nothing ever arrives on: the wait must give up after its limit, set
// the timeout bit of the workspace status word and let the kernel return, so
// that the context stays usable.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ca_internal.h"
#include "sm100_ptx.cuh"

namespace {

__global__ void bounded_wait_selftest_kernel(unsigned int *status, long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ca::mbar_init(&bar, 1);
        abort_flag = 0;
        ca::fence_mbar_init();
    }
    __syncthreads();
    const ca::AbortState ab{&abort_flag, status};
    if (threadIdx.x == 0) {
        // phase 0 never completes: no thread arrives and no copy is in flight
        (void)ca::mbar_wait(&bar, 0, ab, limit_cycles);
    }
    __syncthreads();
}

}  // namespace

extern "C" int ca_selftest_bounded_wait(void *workspace, long long limit_cycles, void *stream) {
    if (!workspace || limit_cycles <= 0 || limit_cycles > ca::kWaitLimitCycles)
        return CA_ERR_INVALID_ARG;
    bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<unsigned int *>(workspace), limit_cycles);
    return cudaGetLastError() == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}
