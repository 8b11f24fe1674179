// selftest.cu -- the bounded-wait path, exercised on purpose.
//
// Every pipeline wait in the library gives up after a time limit, raises the
// timeout code in the device error flag and lets its kernel return, so that a
// lost arrival never hangs the GPU. This kernel makes one such wait run out: a
// CTA waits on an mbarrier that nothing ever arrives on, with the caller's
// limit, and returns. Nothing faults or traps; the context stays usable.
#include "common.cuh"
#include "launch.h"
#include "launch_util.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(32, 1) bounded_wait_kernel(unsigned long long limit_ns, int *err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    griddep_wait();
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, 256, limit_ns);   // no arrival: times out
    __syncwarp();
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(unsigned long long limit_ns, int *err, cudaStream_t s) {
    return launch_pdl(bounded_wait_kernel, dim3(1), dim3(32), 0, s, limit_ns, err);
}

}  // namespace moe
