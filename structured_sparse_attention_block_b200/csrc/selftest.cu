// Timeout self-test of the kernels' bounded waits.  One 32-thread block
// waits, with the library's own mbarrier wait, for a phase of a shared-memory
// barrier that no thread ever arrives on.  The wait gives up after its limit
// (sm100::kWaitLimitNs), records COWA_ERR_TIMEOUT in the device error word,
// raises the block's abort flag (the other threads then stop at once) and the
// kernel returns: the host reads the status through cowa_get_device_error and
// the context stays usable.  No memory outside the block's shared memory is
// touched and no asynchronous copy or tensor-core operation is in flight.
#include "kernels.cuh"
#include "sm100.cuh"

namespace cowa {

using namespace sm100;

__global__ void __launch_bounds__(32) wait_selftest_kernel(int *err)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    // phase 0 never completes: nothing arrives
    mbar_wait(smem_addr(&bar), 0, err, &abort_flag);
}

cudaError_t launch_wait_selftest(int *err, cudaStream_t st)
{
    launch_begin("wait_selftest", st);
    wait_selftest_kernel<<<1, 32, 0, st>>>(err);
    launch_end(st);
    return cudaGetLastError();
}

}  // namespace cowa
