// Failure-path self-test of the bounded device waits.
//
// Every mbarrier wait in the tensor-core kernels gives up after a cycle limit,
// records kStatusTimeout in the device status word and lets its CTA drain and
// exit, so that a lost arrival shows up as PISA_ERR_DEVICE_TIMEOUT on the host
// instead of a hung GPU.  This kernel exercises that path on purpose and
// safely: one thread waits, with a short limit, on a freshly initialised
// mbarrier (one expected arrival) whose first phase nothing ever completes.
// The wait is the one the kernels use (try_wait with a bounded suspend hint,
// then a clock64 check), so it ends after about `limit` cycles; the kernel then
// exits with nothing in flight.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace pisa {

__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(unsigned* status, long long limit) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = tc::smem_addr(&bar);
    tc::mbar_init(b, 1);
    tc::fence_barrier_init();
    bool aborted = false;
    tc::mbar_wait(b, 0, aborted, status, limit);  // phase 0 never completes: times out
}

// Self-test of the two base-2 exponentials the attention kernels use: which = 0
// evaluates the FMA-pipe polynomial tc::ex2_fma, which = 1 the special-function
// unit's ex2.approx, element by element (y[i] = 2^x[i]).
__global__ void ex2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, long long n, int which) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        y[i] = which ? tc::ex2(x[i]) : tc::ex2_fma(x[i]);
}

}  // namespace pisa
