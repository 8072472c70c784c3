// decode.cu -- one recurrent (decode) step for a batch of sequences:
//     state <- exp(dt A_h) state + dt x B^T ;   y = state C + D_h x
// "Transformers are SSMs" (CiteArk), "what this means": constant-memory
// inference; "论文解读：Mamba: ...", 状态空间模型: the linear-recurrence mode
// for autoregressive inference.
//
// The step is pure HBM streaming: every fp32 state element is read once and
// written once, with two flops per byte.  A warp owns kRows consecutive
// state rows (one row = the N-vector of one (batch, head, p)), each lane
// moves 16-byte pieces, and all rows' loads are issued before any arithmetic
// so each warp keeps kRows * 512 bytes in flight.  Loads and stores use the
// streaming cache hints (the state is touched once per step).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kRows = 4;
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

// N % 4 == 0 and N <= 128 * kMaxPieces: each lane handles up to kMaxPieces
// 4-element pieces of each row.
constexpr int kMaxPieces = 2;

template <typename T>
__global__ void __launch_bounds__(kThreads)
step_kernel_v4(float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
               const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
               const float* __restrict__ Dv, T* __restrict__ y, int64_t b, int64_t H, int64_t P,
               int64_t N, int64_t G) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t rows = b * H * P;
    const int64_t hpg = H / G;

    for (int64_t r0 = warp * kRows; r0 < rows; r0 += nwarps * kRows) {
        float s[kRows][kMaxPieces][4];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const int64_t row = r0 + r;
#pragma unroll
            for (int k = 0; k < kMaxPieces; ++k) {
                const int64_t n0 = (int64_t)(k * 32 + lane) * 4;
                if (row < rows && n0 < N) {
                    const float4 q = __ldcs(reinterpret_cast<const float4*>(state + row * N + n0));
                    s[r][k][0] = q.x; s[r][k][1] = q.y; s[r][k][2] = q.z; s[r][k][3] = q.w;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const int64_t row = r0 + r;
            if (row >= rows) break;
            const int64_t bh = row / P;
            const int64_t bb = bh / H, h = bh - bb * H, g = h / hpg;
            const float dtv = dt[bh];
            const float a = expf(dtv * A[h]);
            const float xv = to_f32(x[row]);
            const float u = dtv * xv;
            const T* Bt = Bm + (bb * G + g) * N;
            const T* Ct = Cm + (bb * G + g) * N;
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < kMaxPieces; ++k) {
                const int64_t n0 = (int64_t)(k * 32 + lane) * 4;
                if (n0 < N) {
                    float bv[4], cv[4];
                    load4<T>(Bt + n0, bv);
                    load4<T>(Ct + n0, cv);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        s[r][k][e] = fmaf(a, s[r][k][e], u * bv[e]);
                        acc = fmaf(s[r][k][e], cv[e], acc);
                    }
                    __stcs(reinterpret_cast<float4*>(state + row * N + n0),
                           make_float4(s[r][k][0], s[r][k][1], s[r][k][2], s[r][k][3]));
                }
            }
            acc = warp_sum(acc);
            if (lane == 0) y[row] = from_f32<T>(acc + Dv[h] * xv);
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
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int warps_per_block = kThreads / 32;
    const bool v4 = (d.N % 4 == 0) && (d.N <= 128 * kMaxPieces);
    const int64_t rows_per_block = warps_per_block * (v4 ? kRows : 1);
    int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
    const int64_t cap = (int64_t)sms * 8;  // 8 resident 256-thread blocks per SM
    if (blocks > cap) blocks = cap;
    if (v4) {
        step_kernel_v4<T><<<(unsigned)blocks, kThreads, 0, s>>>(
            state, static_cast<const T*>(x), dt, A, static_cast<const T*>(B),
            static_cast<const T*>(C), D, static_cast<T*>(y), d.b, d.H, d.P, d.N, d.G);
    } else {
        step_kernel_scalar<T><<<(unsigned)blocks, kThreads, 0, s>>>(
            state, static_cast<const T*>(x), dt, A, static_cast<const T*>(B),
            static_cast<const T*>(C), D, static_cast<T*>(y), d.b, d.H, d.P, d.N, d.G);
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
