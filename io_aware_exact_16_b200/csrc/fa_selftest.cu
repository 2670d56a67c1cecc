// fa_selftest.cu -- a check of the failure path every kernel relies on: an mbarrier wait that
// nothing will ever complete gives up after the bounded wait and reports FA_ERR_TIMEOUT
// through the device error flag, leaving the context usable.  No fault, trap or endless loop
// is involved: the wait is the same bounded `mbar_wait` the kernels use.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

__global__ void fa_wait_selftest_kernel(int* err, uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Nothing arrives on this barrier, so its phase 0 never completes.
        const bool done = mbar_wait(&bar, 0, timeout_ns, &abort_flag);
        atomicCAS(err, 0, done ? kErrInvalidArg : kErrTimeout);
    }
}

}  // namespace

cudaError_t launch_wait_selftest(int* err, uint64_t timeout_ns, cudaStream_t stream) {
    fa_wait_selftest_kernel<<<1, 32, 0, stream>>>(err, timeout_ns);
    return cudaGetLastError();
}

}  // namespace fa
