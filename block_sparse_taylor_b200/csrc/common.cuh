// Shared device helpers for the piecewise sparse attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pisa {

typedef __nv_bfloat16 bf16;

// Bits of the device status word (one word per device, read and cleared by
// pisa_poll_device_status).
enum : unsigned {
    kStatusTimeout = 1u,   // a bounded wait on an mbarrier gave up
    kStatusBadShape = 2u,  // a kernel met a shape its launch did not promise
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Canonical fp32 tree sum over N (power of two) register values:
// for h = N/2 .. 1: a[i] = a[i] + a[i+h] (i < h).  Every add is an IEEE
// round-to-nearest fp32 add (no contraction, no reassociation).
template <int N>
__device__ __forceinline__ float tree_sum(float (&a)[N]) {
#pragma unroll
    for (int h = N / 2; h >= 1; h >>= 1) {
#pragma unroll
        for (int i = 0; i < h; ++i) a[i] = __fadd_rn(a[i], a[i + h]);
    }
    return a[0];
}

}  // namespace pisa
