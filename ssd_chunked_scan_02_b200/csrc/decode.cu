// decode.cu -- one recurrent (decode) step for a batch of sequences:
//     state <- exp(dt A_h) state + dt x B^T ;   y = state C + D_h x
// "Transformers are SSMs" (CiteArk), "what this means": constant-memory
// inference; "论文解读：Mamba: ...", 状态空间模型: the linear-recurrence mode
// for autoregressive inference.
//
// The step is pure HBM streaming: every fp32 state element is read once and
// written once, with two flops per byte.  Loads and stores of the state use
// the streaming cache hints (it is touched once per step).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ void load4(const T* p, float* v);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float* v) {
    const float4 q = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&q.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&q.y);
    const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

// One 256-thread block per (batch, head): the head's P x N fp32 state is
// P * N / 4 float4 items; thread t owns items t, t + 256, ... so each warp
// covers whole rows (NV = N / 4 lanes per row, NV a power of two <= 32) and
// always the same four state columns, whose B and C values it loads once.
// dt, A, D and the head's x row are loaded once per block; eight state items
// per thread are loaded before any arithmetic.
template <typename T, int NV>
__global__ void __launch_bounds__(kThreads)
step_kernel_bh(float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
               const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
               const float* __restrict__ Dv, T* __restrict__ y, int64_t H, int64_t P,
               int64_t G) {
    constexpr int N = NV * 4;
    constexpr int kBatch = 8;
    __shared__ float s_x[256];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int64_t bb = bh / H, h = bh - bb * H, g = h / (H / G);
    for (int p = tid; p < P; p += kThreads) s_x[p] = to_f32(x[bh * P + p]);
    const float dtv = dt[bh];
    const float a = expf(dtv * A[h]);
    const float Dh = Dv[h];
    const int n4 = tid % NV;
    float bv[4], cv[4];
    load4<T>(Bm + (bb * G + g) * N + n4 * 4, bv);
    load4<T>(Cm + (bb * G + g) * N + n4 * 4, cv);
    __syncthreads();

    float4* base = reinterpret_cast<float4*>(state + bh * P * N);
    const int items = (int)(P * NV);
    for (int k0 = 0; k0 < items; k0 += kBatch * kThreads) {
        float4 sv[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int it = k0 + k * kThreads + tid;
            if (it < items) sv[k] = __ldcs(base + it);
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int it = k0 + k * kThreads + tid;
            const bool valid = it < items;
            const int p = it / NV;
            float acc = 0.f, xv = 0.f;
            if (valid) {
                xv = s_x[p];
                const float u = dtv * xv;
                float4 q = sv[k];
                q.x = fmaf(a, q.x, u * bv[0]);
                q.y = fmaf(a, q.y, u * bv[1]);
                q.z = fmaf(a, q.z, u * bv[2]);
                q.w = fmaf(a, q.w, u * bv[3]);
                __stcs(base + it, q);
                acc = q.x * cv[0];
                acc = fmaf(q.y, cv[1], acc);
                acc = fmaf(q.z, cv[2], acc);
                acc = fmaf(q.w, cv[3], acc);
            }
#pragma unroll
            for (int o = NV / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (valid && n4 == 0) y[bh * P + p] = from_f32<T>(acc + Dh * xv);
        }
    }
}

// General N (any N <= 256, no vector alignment assumption on rows).
template <typename T>
__global__ void __launch_bounds__(kThreads)
step_kernel_scalar(float* __restrict__ state, const T* __restrict__ x,
                   const float* __restrict__ dt, const float* __restrict__ A,
                   const T* __restrict__ Bm, const T* __restrict__ Cm,
                   const float* __restrict__ Dv, T* __restrict__ y, int64_t b, int64_t H,
                   int64_t P, int64_t N, int64_t G) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t rows = b * H * P;
    const int64_t hpg = H / G;
    for (int64_t row = warp; row < rows; row += nwarps) {
        const int64_t bh = row / P;
        const int64_t bb = bh / H, h = bh - bb * H, g = h / hpg;
        const float dtv = dt[bh];
        const float a = expf(dtv * A[h]);
        const float xv = to_f32(x[row]);
        const float u = dtv * xv;
        float acc = 0.f;
        for (int64_t n = lane; n < N; n += 32) {
            float sv = state[row * N + n];
            sv = fmaf(a, sv, u * to_f32(Bm[(bb * G + g) * N + n]));
            state[row * N + n] = sv;
            acc = fmaf(sv, to_f32(Cm[(bb * G + g) * N + n]), acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) y[row] = from_f32<T>(acc + Dv[h] * xv);
    }
}

template <typename T>
cudaError_t run(float* state, const void* x, const float* dt, const float* A, const void* B,
                const void* C, const float* D, void* y, const Dims& d, cudaStream_t s) {
    const int64_t rows = d.b * d.H * d.P;
    if (rows == 0) return cudaSuccess;
    const T* xp = static_cast<const T*>(x);
    const T* Bp = static_cast<const T*>(B);
    const T* Cp = static_cast<const T*>(C);
    T* yp = static_cast<T*>(y);
    const int64_t bh = d.b * d.H;
    if (d.N == 128 && bh <= 0x7fffffffLL) {
        step_kernel_bh<T, 32><<<(unsigned)bh, kThreads, 0, s>>>(state, xp, dt, A, Bp, Cp, D, yp,
                                                              d.H, d.P, d.G);
    } else if (d.N == 64 && bh <= 0x7fffffffLL) {
        step_kernel_bh<T, 16><<<(unsigned)bh, kThreads, 0, s>>>(state, xp, dt, A, Bp, Cp, D, yp,
                                                              d.H, d.P, d.G);
    } else {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t warps_per_block = kThreads / 32;
        int64_t blocks = (rows + warps_per_block - 1) / warps_per_block;
        const int64_t cap = (int64_t)sms * 8;
        if (blocks > cap) blocks = cap;
        step_kernel_scalar<T><<<(unsigned)blocks, kThreads, 0, s>>>(state, xp, dt, A, Bp, Cp, D, yp,
                                                                   d.b, d.H, d.P, d.N, d.G);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(float* state, const void* x, const float* dt, const float* A,
                        const void* B, const void* C, const float* D, void* y, const Dims& d,
                        Elt t, cudaStream_t s) {
    if (t == Elt::F32) return run<float>(state, x, dt, A, B, C, D, y, d, s);
    return run<__nv_bfloat16>(state, x, dt, A, B, C, D, y, d, s);
}

}  // namespace ssd
