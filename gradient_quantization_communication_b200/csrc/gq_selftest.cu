// gq_selftest.cu -- the failure path of the kernels' bounded waits, exercised without a fault.
//
// Every wait of the kernels for a bulk copy (mbar_wait_warp) gives up after a time limit and
// raises the plan's timeout flag instead of hanging.  This kernel waits with that same function
// on an mbarrier whose phase nothing ever completes (no thread arrives, no copy is issued), so
// the wait runs out, the flag is raised and the kernel returns normally.
#include "gq_device.cuh"

namespace gq {
namespace {

__global__ void __launch_bounds__(32) k_wait_selftest(unsigned int *status, unsigned long long limit_ns)
{
    __shared__ unsigned long long bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected, none will come
        fence_barrier_init();
    }
    __syncwarp();
    if (!mbar_wait_warp(&bar, 0u, limit_ns) && threadIdx.x == 0) atomicOr(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned int *status, unsigned long long limit_ns, cudaStream_t stream)
{
    k_wait_selftest<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace gq
