// kda_selftest.cu -- device-side self-test of the time-limited waits.
//
// Every wait in the libkda kernels (TMA and tensor-core completion on an
// mbarrier) gives up after a clock limit and records KDA_ERR_TIMEOUT in the
// device status word instead of hanging.  This kernel exercises exactly that
// path on an mbarrier that nothing ever arrives on, with a short limit, so a
// test can check that the status is reported and that the context stays usable.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tc.cuh"

namespace kda {

__global__ void wait_selftest_kernel(int *status, long long limit_cycles) {
    __shared__ __align__(8) uint64_t mbar;
    const uint32_t m = smem_u32(&mbar);
    if (threadIdx.x == 0) tc::mbar_init(m, 1);
    __syncthreads();
    if (threadIdx.x == 0 && !tc::mbar_wait(m, 0u, limit_cycles)) atomicExch(status, kStatusTimeout);
}

cudaError_t launch_wait_selftest(int *status, long long limit_cycles, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_cycles);
    return cudaGetLastError();
}

}  // namespace kda
