// Self-test of the failure path that every kernel of this library shares: a bounded mbarrier wait
// that runs out records PA_ERR_TIMEOUT in the status word and the kernel returns, so the context
// stays usable and the host reads the error.  The barrier waited on here is one that nothing ever
// arrives on; the wait is bounded by %globaltimer like every other wait of the library.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

__global__ void __launch_bounds__(32) pa_wait_timeout_kernel(int32_t *status, uint64_t timeout_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    // phase 0 never completes: no thread arrives and no copy is attached to the barrier
    const bool done = mbar_wait(&bar, 0, timeout_ns);
    if (!__any_sync(0xffffffffu, done) && threadIdx.x == 0)
        set_status(status, PA_ERR_TIMEOUT);
}

}  // namespace pa

using namespace pa;

extern "C" int pa_selftest_wait_timeout(int32_t *status, uint64_t timeout_ns, void *stream)
{
    CallRange range(__func__);
    if (!aligned4(status) || timeout_ns == 0 || timeout_ns > 100000000ull)
        return PA_ERR_ARG;
    pa_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, timeout_ns);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
