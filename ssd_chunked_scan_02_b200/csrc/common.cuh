// common.cuh -- small device helpers shared by the SSD kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Inclusive prefix sum of a[0..n) in shared memory, done by warp 0 in
// 32-element pieces (n <= a few hundred).  The caller synchronises the block
// before and after.
__device__ __forceinline__ void warp0_inclusive_scan(float* a, int n) {
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    float carry = 0.f;
    for (int base = 0; base < n; base += 32) {
        float v = (base + lane < n) ? a[base + lane] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        v += carry;
        if (base + lane < n) a[base + lane] = v;
        carry = __shfl_sync(0xffffffffu, v, 31);
    }
}

}  // namespace ssd
