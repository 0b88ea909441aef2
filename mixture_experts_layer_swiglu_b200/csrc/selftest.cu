// selftest.cu -- a check of the library's bounded waits.
//
// Every wait in the kernels (on an mbarrier fed by TMA copies, MMA commits or
// other warps) gives up after a time limit, records MOE_ERR_TIMEOUT in the
// device status word and lets the kernel return, so a fault elsewhere cannot
// hang the GPU.  moe_selftest_wait_timeout() runs that wait on a barrier that
// nothing ever arrives on, with a short limit: the kernel must return and the
// status must read MOE_ERR_TIMEOUT, with the CUDA context still usable.

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__global__ void wait_never_kernel(uint64_t limit_ns, int* waited_ok)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);                 // one arrival expected; none comes
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) *waited_ok = mbar_wait(&bar, 0, limit_ns) ? 1 : 0;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API moe_status moe_selftest_wait_timeout(uint64_t limit_ns, int32_t* waited_ok, moe_stream_t stream)
{
    t_launches = 0;
    if (!waited_ok || limit_ns == 0 || limit_ns > kWaitLimitNs) return MOE_ERR_INVALID_ARG;
    wait_never_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, waited_ok);
    count_launch();
    return cuda_status(cudaGetLastError());
}
