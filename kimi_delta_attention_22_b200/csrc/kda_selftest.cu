// kda_selftest.cu -- failure detection without a GPU fault: one CTA takes the
// same bounded mbarrier wait (sm100::mbar_wait) as the tensor-core kernels, on
// a barrier of its own that either completes or never does, and reports an
// expiry through the status word the way those kernels do.  Nothing is in
// flight while it waits, so an expiry leaves the context as it was.
#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

__global__ void __launch_bounds__(128, 1) kda_selftest_wait_kernel(int32_t* dev_status, uint64_t budget_ns,
                                                                    int complete) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (complete && threadIdx.x == 0) mbar_arrive(&bar);
    // phase 0 completes only through the arrival above
    const bool ok = mbar_wait(&bar, 0, budget_ns);
    if (__syncthreads_or(!ok) && threadIdx.x == 0) atomicOr(dev_status, KDA_DEV_TIMEOUT);
}

}  // namespace

cudaError_t launch_selftest_wait(int32_t* dev_status, uint64_t budget_ns, bool complete, cudaStream_t s) {
    kda_selftest_wait_kernel<<<1, 128, 0, s>>>(dev_status, budget_ns, complete ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace kda
