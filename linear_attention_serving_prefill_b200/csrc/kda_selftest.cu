// Failure-detection self-test: one CTA waits on an mbarrier that nothing
// completes, with the same bounded-wait primitive the tensor-core kernels use.
// The wait gives up after `limit_ns`, records the timeout in the device status
// word and the kernel returns normally -- no trap, no fault, no hang -- so the
// host reads the status and the context stays usable.
#include "kda_internal.h"
#include "kda_prefill_tc.h"
#include "tc_ptx.cuh"

namespace kda {
namespace {

__global__ void wait_timeout_selftest_kernel(int32_t *status, int64_t limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);  // expects one arrival that never comes
        tc::fence_mbar_init();
    }
    __syncthreads();
    const bool done = tc::mbar_wait(&bar, 0, tc::globaltimer_ns() + (uint64_t)limit_ns);
    if (!done && threadIdx.x == 0) atomicCAS(status, 0, (int32_t)KDA_TC_TIMEOUT_CODE);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(int32_t *status, int64_t limit_ns, cudaStream_t stream)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace kda
