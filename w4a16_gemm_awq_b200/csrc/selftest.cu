// selftest.cu -- exercises the bounded-wait path that every pipeline wait in the kernels uses.
//
// One thread initialises an mbarrier that nothing will ever complete, then waits on it with
// the same try-wait / global-timer loop as the kernels, but with a caller-given limit.  The
// wait runs out, the kernel records kErrTimeout in the device status word and returns; the
// context stays usable.  No trap, assert or fault is involved.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {

__global__ void selftest_timeout_kernel(unsigned long long limit_ns, unsigned* err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);  // one arrival expected, none ever made
    fence_mbarrier_init();
    const unsigned long long t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait(&bar, 0)) return;  // cannot happen: the phase never completes
        if (global_timer_ns() - t0 > limit_ns) {
            record_error(err, kErrTimeout);
            return;
        }
    }
}

cudaError_t launch_selftest_timeout(unsigned long long limit_ns, unsigned* err, cudaStream_t stream) {
    selftest_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
    return cudaGetLastError();
}

}  // namespace w4a16
