// selftest.cu -- a kernel whose only job is to let a bounded wait run out.
//
// Every producer/consumer handshake of the layer kernels waits through mbar_wait, which gives up
// after a fixed number of SM clock cycles, records MOE_ERR_TIMEOUT in the call's status words and
// lets the kernel finish instead of spinning forever.  This kernel waits, with the same helper and
// a short limit, on an mbarrier that nothing ever arrives on, so a test can check that the give-up
// path reports the status and leaves the context usable.  It faults nothing and ends by itself
// (no copy is in flight, the barrier lives in its own shared memory).
#include "common.cuh"

namespace moe {

constexpr long long kSelfTestWaitCycles = 20000000LL;   // ~10 ms at 2 GHz

__global__ void wait_timeout_selftest_kernel(int32_t *status_out)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const StatusPtrs st{nullptr, status_out};
    bool aborted = false;
    mbar_wait<kSelfTestWaitCycles>(&bar, 0, aborted, st);   // nothing arrives: gives up
    mbar_wait<kSelfTestWaitCycles>(&bar, 0, aborted, st);   // after giving up, returns at once
    __syncthreads();                                        // every thread got past both waits
}

cudaError_t launch_wait_timeout_selftest(int32_t *status_out, cudaStream_t s)
{
    wait_timeout_selftest_kernel<<<1, 64, 0, s>>>(status_out);
    return cudaGetLastError();
}

}  // namespace moe
