// Self-test of the GEMM kernels' error path on the device: one thread waits,
// through the same bounded mbarrier wait the pipeline roles use, on a barrier
// that nothing arrives on.  The wait gives up after the given time, raises
// the abort flag and the DEVERR_TIMEOUT status bit, and the kernel returns:
// nothing faults, traps or hangs, and the host reads the status word.
#include <cuda_runtime.h>

#include "kernel.cuh"
#include "launch.h"

namespace fp8nt {

namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_selftest_kernel(unsigned int *status,
                                                                       unsigned long long timeout_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0u;
        fence_mbarrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        Params p{};
        p.status = status;
        p.timeout_ns = timeout_ns;
        // phase 0 of a barrier with one pending arrival never completes
        const bool done = wait_bar(&bar, 0u, &abort_flag, p);
        if (done) // cannot happen; report it as a bad result rather than silently
            atomicOr(status, DEVERR_BAD_INDEX);
    }
}

} // namespace

cudaError_t launch_wait_timeout_selftest(unsigned int *status, unsigned long long timeout_ns,
                                         cudaStream_t stream)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
    return cudaGetLastError();
}

} // namespace fp8nt
