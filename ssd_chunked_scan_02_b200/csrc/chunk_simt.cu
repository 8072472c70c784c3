// chunk_simt.cu -- SIMT (CUDA-core, exact fp32 arithmetic) versions of the
// chunk-local steps of the block-decomposed SSD forward.
//
// They serve the fp32 dtype (whose 1e-4 accuracy target rules out tf32 tensor
// cores) and every shape the tensor-core kernels do not cover.  Both kernels
// work on one (batch, chunk, head) per CTA.
//
// Notation (per chunk, per head h, token offsets i, j inside the chunk):
//   cs_t  = sum_{k <= t} dt_k A_h                       (inclusive prefix of dt*A)
//   chunk state  S = sum_j exp(cs_last - cs_j) dt_j x_j B_j^T
//   output       y_i = sum_{j <= i} (C_i . B_j) exp(cs_i - cs_j) dt_j x_j     (masked C B^T term)
//                    + exp(cs_i) h_prev C_i + D_h x_i                          (entering state + skip)
// "Transformers are SSMs" (CiteArk), AI research summary (block-decomposed
// semiseparable matrix), and the review page's 核心概念 items 2, 3, 5
// (semiseparable matrix; structured masked attention; SSD block algorithm).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kJT = 32;    // tokens per staged j-tile
constexpr int kIT = 16;    // output rows per i-tile
constexpr int kOPT = 8;    // chunk-state outputs per thread per pass
constexpr int kMaxOutPerThread = (kIT * 256 + kThreads - 1) / kThreads;  // P <= 256

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_state_simt_kernel(const T* __restrict__ x, const float* __restrict__ dt,
                        const float* __restrict__ A, const T* __restrict__ Bm,
                        float* __restrict__ states, float* __restrict__ logdecay, Dims d) {
    const int64_t bt = blockIdx.x;
    const int64_t c = bt % d.T, bb = bt / d.T;
    const int h = blockIdx.y;
    const int P = (int)d.P, N = (int)d.N, Q = d.Q;
    const int64_t H = d.H, G = d.G, L = d.L;
    const int64_t g = h / (H / G);
    const int64_t t0 = c * Q;
    const int len = (int)((L - t0) < Q ? (L - t0) : Q);

    extern __shared__ float sm[];
    float* cs = sm;                 // Q
    float* w = cs + Q;              // Q
    float* xs = w + Q;              // kJT * P
    float* bs = xs + kJT * P;       // kJT * N

    const float Ah = A[h];
    for (int t = threadIdx.x; t < len; t += kThreads) cs[t] = dt[(bb * L + t0 + t) * H + h] * Ah;
    __syncthreads();
    warp0_inclusive_scan(cs, len);
    __syncthreads();
    const float last = cs[len - 1];
    for (int t = threadIdx.x; t < len; t += kThreads)
        w[t] = expf(last - cs[t]) * dt[(bb * L + t0 + t) * H + h];
    if (threadIdx.x == 0) logdecay[(bb * d.T + c) * H + h] = last;
    __syncthreads();

    const int PN = P * N;
    float* out = states + ((bb * d.T + c) * H + h) * (int64_t)PN;
    for (int o0 = 0; o0 < PN; o0 += kThreads * kOPT) {
        float acc[kOPT];
#pragma unroll
        for (int k = 0; k < kOPT; ++k) acc[k] = 0.f;
        for (int j0 = 0; j0 < len; j0 += kJT) {
            const int jn = min(kJT, len - j0);
            for (int e = threadIdx.x; e < jn * P; e += kThreads) {
                const int jj = e / P, p = e - jj * P;
                xs[e] = w[j0 + jj] * to_f32(x[((bb * L + t0 + j0 + jj) * H + h) * P + p]);
            }
            for (int e = threadIdx.x; e < jn * N; e += kThreads) {
                const int jj = e / N, n = e - jj * N;
                bs[e] = to_f32(Bm[((bb * L + t0 + j0 + jj) * G + g) * N + n]);
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kOPT; ++k) {
                const int o = o0 + k * kThreads + threadIdx.x;
                if (o < PN) {
                    const int p = o / N, n = o - p * N;
                    float a = acc[k];
                    for (int jj = 0; jj < jn; ++jj) a = fmaf(xs[jj * P + p], bs[jj * N + n], a);
                    acc[k] = a;
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int k = 0; k < kOPT; ++k) {
            const int o = o0 + k * kThreads + threadIdx.x;
            if (o < PN) out[o] = acc[k];
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_out_simt_kernel(const T* __restrict__ x, const float* __restrict__ dt,
                      const float* __restrict__ A, const T* __restrict__ Bm,
                      const T* __restrict__ Cm, const float* __restrict__ Dv,
                      const T* __restrict__ prev, T* __restrict__ y, Dims d) {
    const int64_t bt = blockIdx.x;
    const int64_t c = bt % d.T, bb = bt / d.T;
    const int h = blockIdx.y;
    const int P = (int)d.P, N = (int)d.N, Q = d.Q;
    const int64_t H = d.H, G = d.G, L = d.L;
    const int64_t g = h / (H / G);
    const int64_t t0 = c * Q;
    const int len = (int)((L - t0) < Q ? (L - t0) : Q);
    const int NB = N + 1;  // padded row stride of the staged B tile (bank-conflict free)

    extern __shared__ float sm[];
    float* cs = sm;                   // Q
    float* dts = cs + Q;              // Q
    float* ct = dts + Q;              // kIT * N
    float* bj = ct + kIT * N;         // kJT * (N + 1)
    float* xj = bj + kJT * NB;        // kJT * P
    float* gs = xj + kJT * P;         // kIT * kJT
    float* hs = gs + kIT * kJT;       // P * 33

    const float Ah = A[h];
    for (int t = threadIdx.x; t < len; t += kThreads) {
        const float v = dt[(bb * L + t0 + t) * H + h];
        dts[t] = v;
        cs[t] = v * Ah;
    }
    __syncthreads();
    warp0_inclusive_scan(cs, len);
    __syncthreads();

    const T* hp = prev + ((bb * d.T + c) * H + h) * (int64_t)P * N;
    const float Dh = Dv[h];

    for (int i0 = 0; i0 < len; i0 += kIT) {
        const int in = min(kIT, len - i0);
        for (int e = threadIdx.x; e < in * N; e += kThreads) {
            const int ii = e / N, n = e - ii * N;
            ct[e] = to_f32(Cm[((bb * L + t0 + i0 + ii) * G + g) * N + n]);
        }
        float acc[kMaxOutPerThread];
#pragma unroll
        for (int k = 0; k < kMaxOutPerThread; ++k) acc[k] = 0.f;

        const int jend = i0 + in;  // causal: j <= i < i0 + in
        for (int j0 = 0; j0 < jend; j0 += kJT) {
            const int jn = min(kJT, jend - j0);
            for (int e = threadIdx.x; e < jn * N; e += kThreads) {
                const int jj = e / N, n = e - jj * N;
                bj[jj * NB + n] = to_f32(Bm[((bb * L + t0 + j0 + jj) * G + g) * N + n]);
            }
            for (int e = threadIdx.x; e < jn * P; e += kThreads) {
                const int jj = e / P, p = e - jj * P;
                xj[e] = to_f32(x[((bb * L + t0 + j0 + jj) * H + h) * P + p]);
            }
            __syncthreads();
            for (int e = threadIdx.x; e < kIT * kJT; e += kThreads) {
                const int ii = e / kJT, jj = e - ii * kJT;
                const int i = i0 + ii, j = j0 + jj;
                float v = 0.f;
                if (ii < in && jj < jn && j <= i) {
                    float dot = 0.f;
                    for (int n = 0; n < N; ++n) dot = fmaf(ct[ii * N + n], bj[jj * NB + n], dot);
                    v = dot * expf(cs[i] - cs[j]) * dts[j];
                }
                gs[e] = v;
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kMaxOutPerThread; ++k) {
                const int o = k * kThreads + threadIdx.x;
                if (o < in * P) {
                    const int ii = o / P, p = o - ii * P;
                    float a = acc[k];
                    for (int jj = 0; jj < jn; ++jj) a = fmaf(gs[ii * kJT + jj], xj[jj * P + p], a);
                    acc[k] = a;
                }
            }
            __syncthreads();
        }

        // entering-state term: s(i, p) = sum_n C[i, n] h_prev[p, n]
        float sacc[kMaxOutPerThread];
#pragma unroll
        for (int k = 0; k < kMaxOutPerThread; ++k) sacc[k] = 0.f;
        for (int n0 = 0; n0 < N; n0 += 32) {
            const int nn_n = min(32, N - n0);
            for (int e = threadIdx.x; e < P * 32; e += kThreads) {
                const int p = e >> 5, nn = e & 31;
                hs[p * 33 + nn] = (nn < nn_n) ? to_f32(hp[(int64_t)p * N + n0 + nn]) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kMaxOutPerThread; ++k) {
                const int o = k * kThreads + threadIdx.x;
                if (o < in * P) {
                    const int ii = o / P, p = o - ii * P;
                    float a = sacc[k];
                    for (int nn = 0; nn < nn_n; ++nn) a = fmaf(ct[ii * N + n0 + nn], hs[p * 33 + nn], a);
                    sacc[k] = a;
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int k = 0; k < kMaxOutPerThread; ++k) {
            const int o = k * kThreads + threadIdx.x;
            if (o < in * P) {
                const int ii = o / P, p = o - ii * P;
                const int i = i0 + ii;
                const int64_t xi = ((bb * L + t0 + i) * H + h) * P + p;
                const float xv = to_f32(x[xi]);
                const float v = acc[k] + expf(cs[i]) * sacc[k] + Dh * xv;
                y[xi] = from_f32<T>(v);
            }
        }
        __syncthreads();
    }
}

size_t state_smem(const Dims& d) { return sizeof(float) * (2 * d.Q + kJT * (d.P + d.N)); }
size_t out_smem(const Dims& d) {
    return sizeof(float) *
           (2 * d.Q + kIT * d.N + kJT * (d.N + 1) + kJT * d.P + kIT * kJT + d.P * 33);
}

template <typename T>
cudaError_t state_impl(const void* x, const float* dt, const float* A, const void* B,
                       float* states, float* logdecay, const Dims& d, cudaStream_t s) {
    const size_t smem = state_smem(d);
    cudaError_t e = cudaFuncSetAttribute(chunk_state_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(d.b * d.T), (unsigned)d.H);
    chunk_state_simt_kernel<T><<<grid, kThreads, smem, s>>>(
        static_cast<const T*>(x), dt, A, static_cast<const T*>(B), states, logdecay, d);
    return cudaGetLastError();
}

template <typename T>
cudaError_t out_impl(const void* x, const float* dt, const float* A, const void* B, const void* C,
                     const float* D, const void* prev, void* y, const Dims& d, cudaStream_t s) {
    const size_t smem = out_smem(d);
    cudaError_t e = cudaFuncSetAttribute(chunk_out_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(d.b * d.T), (unsigned)d.H);
    chunk_out_simt_kernel<T><<<grid, kThreads, smem, s>>>(
        static_cast<const T*>(x), dt, A, static_cast<const T*>(B), static_cast<const T*>(C), D,
        static_cast<const T*>(prev), static_cast<T*>(y), d);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_state_simt(const void* x, const float* dt, const float* A, const void* B,
                                    float* states, float* logdecay, const Dims& d, Elt t,
                                    cudaStream_t s) {
    if (t == Elt::F32) return state_impl<float>(x, dt, A, B, states, logdecay, d, s);
    return state_impl<__nv_bfloat16>(x, dt, A, B, states, logdecay, d, s);
}

cudaError_t launch_chunk_out_simt(const void* x, const float* dt, const float* A, const void* B,
                                  const void* C, const float* D, const void* prev, void* y,
                                  const Dims& d, Elt t, cudaStream_t s) {
    if (t == Elt::F32) return out_impl<float>(x, dt, A, B, C, D, prev, y, d, s);
    return out_impl<__nv_bfloat16>(x, dt, A, B, C, D, prev, y, d, s);
}

}  // namespace ssd
