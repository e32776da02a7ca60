// Failure-handling self-test: one CTA waits, through the same bounded
// mbarrier wait every tensor-core kernel of the library uses, on a barrier
// that no thread ever arrives on.  The wait gives up after the caller's cycle
// limit and records the timeout in the device error word, exactly as a
// stalled kernel would; nothing faults, traps or spins without end, so the
// CUDA context stays usable.
#include "tcgen05.cuh"

namespace scope {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(int32_t *err, long long limit)
{
    __shared__ uint64_t never;  // initialised for one arrival that never comes
    __shared__ int abort_sh;
    if (threadIdx.x == 0) {
        tc::mbar_init(&never, 1);
        abort_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    tc::mbar_wait_limit(&never, 0, &abort_sh, err, 0x7E, limit);
}

}  // namespace

void launch_wait_timeout(int32_t *err, long long limit, cudaStream_t st)
{
    wait_timeout_kernel<<<1, 32, 0, st>>>(err, limit);
    count_launches(1);
}

}  // namespace scope
