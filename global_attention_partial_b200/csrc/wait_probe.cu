// Test probe of the bounded pipeline wait.
//
// One warp initialises an mbarrier that nothing ever arrives on and waits for
// it with mbar_wait, the wait every pipelined kernel of the library uses. The
// wait runs into the device's wait limit, sets the timeout bit of the device
// error word and returns; the kernel then exits normally. Nothing is in
// flight (no copy, no tensor-core operation), so the timeout leaves the
// context usable. Only the library's debug entry point launches it, with the
// limit shortened beforehand through the matching test hook.
#include "kernels.cuh"

namespace mimo {
namespace {

__global__ void wait_probe_kernel(unsigned *err)
{
    __shared__ uint64_t bar;
    __shared__ int stop;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        stop = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        mbar_wait(&bar, 0, &stop, err);  // no arrival: ends at the wait limit
    __syncthreads();
}

} // namespace

cudaError_t launch_wait_probe(unsigned *err, cudaStream_t stream)
{
    wait_probe_kernel<<<1, 32, 0, stream>>>(err);
    return cudaGetLastError();
}

} // namespace mimo
