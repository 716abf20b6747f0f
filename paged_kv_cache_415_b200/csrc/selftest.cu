// selftest.cu -- pa_selftest_bounded_wait: the library's bounded mbarrier
// wait (pa_common.cuh) made to run out on purpose, on a barrier that nothing
// arrives on.  Declared in pa_selftest.h; for tests only.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"
#include "pa_common.cuh"
#include "pa_host.h"
#include "pa_selftest.h"

namespace pa {

__global__ void __launch_bounds__(128) selftest_bounded_wait_kernel(int32_t* d_status,
                                                                    int64_t* d_wait_ns,
                                                                    uint32_t limit_us)
{
    __shared__ uint64_t never;               // no thread and no copy ever arrives on it
    if (threadIdx.x == 0) {
        mbar_init(&never, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const uint64_t t0 = global_timer_ns();
    const bool completed = mbar_wait_warp(&never, 0u, 1000ull * limit_us);
    const uint64_t waited = global_timer_ns() - t0;
    if (!completed && (threadIdx.x & 31) == 0) status_or(d_status, PA_STATUS_TIMEOUT);
    // the CTA's measured wait: the shortest over its warps
    __shared__ unsigned long long shortest;
    if (threadIdx.x == 0) shortest = ~0ull;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) atomicMin(&shortest, static_cast<unsigned long long>(waited));
    __syncthreads();
    if (threadIdx.x == 0 && d_wait_ns != nullptr)
        d_wait_ns[blockIdx.x] = static_cast<int64_t>(shortest);
}

}  // namespace pa

extern "C" pa_status pa_selftest_bounded_wait(int32_t* d_status, int64_t* d_wait_ns,
                                              uint32_t wait_limit_us, int32_t num_ctas,
                                              pa_stream_t stream)
{
    using namespace pa;
    if (d_status == nullptr || !aligned4(d_status) || (d_wait_ns && !aligned8(d_wait_ns)))
        return PA_ERR_INVALID_ARG;
    if (wait_limit_us == 0u || wait_limit_us > 1000000u || num_ctas < 1 || num_ctas > 1024)
        return PA_ERR_INVALID_ARG;
    selftest_bounded_wait_kernel<<<num_ctas, 128, 0, stream>>>(d_status, d_wait_ns,
                                                               wait_limit_us);
    return launch_status();
}
