// Device-side check of the bounded waits that the tensor-core prefill relies on for
// failure detection: one thread waits on an mbarrier with the same helper and time
// limit logic as the prefill's waits.  With `arrive` set the barrier's phase completes
// and the wait succeeds; without it nothing ever arrives, the wait gives up after
// limit_ns and the kernel records the timeout in the status word (bit 0, read on the
// host as KDA_ERR_TIMEOUT) and returns, leaving the context usable.  No fault, trap or
// unbounded loop is involved.
#include "kernels.h"
#include "tc_ptx.cuh"

namespace kda {

namespace {

__global__ void kda_bounded_wait_selftest_kernel(int arrive, unsigned long long limit_ns, unsigned int *status)
{
    __shared__ __align__(8) unsigned long long bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = ptx::smem_u32(&bar);
    ptx::mbar_init(b, 1);
    ptx::fence_mbar_init();
    if (arrive) ptx::mbar_arrive(b);
    if (!ptx::mbar_wait(b, 0, limit_ns)) atomicOr(status, 1u);
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int arrive, unsigned long long limit_ns, unsigned int *status,
                                         cudaStream_t stream)
{
    kda_bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(arrive, limit_ns, status);
    return cudaGetLastError();
}

}  // namespace kda
