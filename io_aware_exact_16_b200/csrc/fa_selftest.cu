// fa_selftest.cu -- checks of the failure paths every kernel relies on.
//   wait:   an mbarrier wait that nothing will ever complete gives up after the bounded wait and
//           reports FA_ERR_TIMEOUT through the device error flag, leaving the context usable.
//           No fault, trap or endless loop is involved: the wait is the same bounded
//           `mbar_wait` the kernels use.
//   bounds: (FA_DEBUG builds) the index check every plain global access of the kernels goes
//           through, given one index inside and one just past a caller's buffer: the first
//           store happens, the second is skipped and reported as FA_ERR_INVALID_ARG.
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

// One thread: a checked store of `value` to buf[n - 1] (inside) and to buf[n] (one past the
// end).  With the checks compiled in, only the first happens.
__global__ void fa_bounds_selftest_kernel(int* buf, int n, int value, int* err) {
    if (threadIdx.x != 0) return;
    for (int i = n - 1; i <= n; ++i)
        if (in_bounds(err, (size_t)i, 1, (size_t)n)) buf[i] = value;
}

}  // namespace

cudaError_t launch_bounds_selftest(int* buf, int n, int value, int* err, cudaStream_t stream) {
    fa_bounds_selftest_kernel<<<1, 32, 0, stream>>>(buf, n, value, err);
    return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int* err, uint64_t timeout_ns, cudaStream_t stream) {
    fa_wait_selftest_kernel<<<1, 32, 0, stream>>>(err, timeout_ns);
    return cudaGetLastError();
}

}  // namespace fa
