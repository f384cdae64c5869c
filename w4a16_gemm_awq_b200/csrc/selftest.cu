// selftest.cu -- on-device checks of two mechanisms the kernels rely on.
//
// Bounded waits: one thread initialises an mbarrier that nothing will ever complete, then
// waits on it with the same try-wait / global-timer loop as the kernels, but with a
// caller-given limit.  The wait runs out, the kernel records kErrTimeout in the device status
// word and returns; the context stays usable.  No trap, assert or fault is involved.
//
// The quantizer's division: quotient_markstein against the IEEE division (__fdiv_rn) for
// every divisor with an 11-bit significand (every fp16 value, up to a power of two) and every
// dividend significand, both signs, with quotients of magnitude 2^-4 .. 2^7 (where the 4-bit
// code depends on the rounding; beyond that it saturates, below it rounds to 0 either way).
// Both operations are exact functions of the operands' significands as long as nothing
// overflows or underflows, so a divisor in [1, 2) and dividends in [2^-3, 2^7) cover the
// domain.
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

// blockIdx.y: divisor b = 1 + j / 1024; dividends a = +-(1 + m 2^-23) 2^e, e = -3 .. 6.
__global__ void __launch_bounds__(256) selftest_quotient_kernel(unsigned long long* mismatches,
                                                               unsigned* first /* [4]: b bits, a bits, got, want */) {
    const float b = 1.0f + (float)blockIdx.y * (1.0f / 1024.0f);
    const float y = __frcp_rn(b);
    unsigned long long bad = 0;
    for (uint32_t m = blockIdx.x * 256 + threadIdx.x; m < (1u << 23); m += gridDim.x * 256) {
#pragma unroll 2
        for (int e = -3; e <= 6; ++e) {
#pragma unroll
            for (int sg = 0; sg < 2; ++sg) {
                const float a = __uint_as_float(((uint32_t)sg << 31) | ((uint32_t)(127 + e) << 23) | m);
                const float got = quotient_markstein(a, b, y);
                const float want = __fdiv_rn(a, b);
                if (__float_as_uint(got) != __float_as_uint(want)) {
                    ++bad;
                    if (atomicCAS(first, 0u, __float_as_uint(b)) == 0u) {
                        first[1] = __float_as_uint(a);
                        first[2] = __float_as_uint(got);
                        first[3] = __float_as_uint(want);
                    }
                }
            }
        }
    }
    if (bad) atomicAdd(mismatches, bad);
}

cudaError_t launch_selftest_quotient(unsigned long long* mismatches, unsigned* first, cudaStream_t stream) {
    selftest_quotient_kernel<<<dim3(256, 1024), 256, 0, stream>>>(mismatches, first);
    return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(unsigned long long limit_ns, unsigned* err, cudaStream_t stream) {
    selftest_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
    return cudaGetLastError();
}

}  // namespace w4a16
