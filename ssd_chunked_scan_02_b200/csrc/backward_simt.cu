// backward_simt.cu -- gradients of the SSD layer: a first, exact fp32 version
// on the CUDA cores.
//
// "Transformers are SSMs" (CiteArk), AI research summary: training is what the
// layer is for; the gradients are the chain rule applied to the recurrence
//
//     a_t = exp(dt_t A_h),   S_t = a_t S_{t-1} + dt_t x_t B_t^T,   y_t = S_t C_t + D_h x_t
//
// in reverse token order.  With G = dL/dS_t (starting at dL/dfinal, plus
// dy_t C_t^T at every token):
//     dx_t = D_h dy_t + dt_t G B_t          dB_t += dt_t G^T x_t      dC_t += S_t^T dy_t
//     ddt_t = x_t^T G B_t + A_h a_t <G, S_{t-1}>      dA_h += dt_t a_t <G, S_{t-1}>
//     dD_h += dy_t . x_t,   then G <- a_t G;   dinit = G after token 0.
//
// The rows p of a state evolve independently (S_t[p] = a_t S_{t-1}[p] + dt_t
// x_t[p] B_t); only sums couple them.  So one CTA takes a block of R rows of
// one (batch, head) -- R N <= 1024 state elements, 8 a thread -- and walks the
// sequence: a forward sweep stores its rows of the fp32 state every kSeg
// tokens (checkpoints); the reverse sweep recomputes each segment's states
// from its checkpoint into scratch and walks them backwards.  Small CTAs let
// several share an SM and hide each other's memory latency.  dB, dC, ddt, dA
// and dD are sums over rows (and over a group's heads, or the batch): they are
// accumulated atomically into outputs the host zeroes first, so their
// summation order (not their value) varies from run to run.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kBwdThreads = 128;
constexpr int kSeg = 64;          // tokens per checkpoint segment
constexpr int kMaxPer = 8;        // state elements per thread
constexpr int kElems = kBwdThreads * kMaxPer;   // state elements per CTA

__host__ __device__ __forceinline__ int64_t bwd_segments(int64_t L) { return (L + kSeg - 1) / kSeg; }
// rows of the state per CTA, and row blocks per (batch, head)
__host__ __device__ __forceinline__ int bwd_rows(int P, int N) {
    const int r = kElems / N;
    return r < P ? r : P;
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
ssd_bwd_kernel(const T* __restrict__ x, const float* __restrict__ dt, const float* __restrict__ A,
               const T* __restrict__ Bm, const T* __restrict__ Cm, const float* __restrict__ Dv,
               const float* __restrict__ init, const T* __restrict__ dy,
               const float* __restrict__ dfinal, float* __restrict__ dx, float* __restrict__ ddt,
               float* __restrict__ dA, float* __restrict__ dB, float* __restrict__ dC,
               float* __restrict__ dD, float* __restrict__ dinit, float* __restrict__ ws, Dims d) {
    const int64_t H = d.H, G = d.G, L = d.L;
    const int P = (int)d.P, N = (int)d.N, PN = P * N;
    const int R = bwd_rows(P, N);
    const int nrb = (P + R - 1) / R;
    const int64_t bh = blockIdx.x / nrb;
    const int rb_i = (int)(blockIdx.x - bh * nrb);
    const int64_t b = bh / H;
    const int h = (int)(bh % H);
    const int64_t g = h / (H / G);
    const int p0 = rb_i * R;
    const int rows = (P - p0) < R ? (P - p0) : R;
    const int E = rows * N;                              // this CTA's state elements
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t nseg = bwd_segments(L);
    float* ck = ws + (int64_t)blockIdx.x * (nseg + kSeg) * (R * N);   // checkpoint s: before token s kSeg
    float* sg = ck + nseg * (R * N);                                   // states of one segment
    const int64_t soff = bh * PN + (int64_t)p0 * N;                   // rows p0.. of a (b,H,P,N) state

    extern __shared__ float sm[];
    float* sx = sm;              // R   x_t rows
    float* sdy = sx + R;         // R   dy_t rows
    float* rx = sdy + R;         // R   sum_n G[p][n] B_t[n]
    float* sB = rx + R;          // N   B_t
    float* sC = sB + N;          // N   C_t
    float* rbs = sC + N;         // N   sum_p G[p][n] x_t[p]
    float* rcs = rbs + N;        // N   sum_p S_t[p][n] dy_t[p]
    float* sw = rcs + N;         // 2 x 4 warp partials

    const float Ah = A[h], Dh = Dv[h];
    const bool warp_rows = (N % 32) == 0;        // then a warp's 32 elements share a row
    float S[kMaxPer], Gm[kMaxPer];
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        const int e = tid + kBwdThreads * k;
        S[k] = (e < E && init) ? init[soff + e] : 0.f;
        Gm[k] = (e < E && dfinal) ? dfinal[soff + e] : 0.f;
    }
    auto stage_xb = [&](int64_t t) {
        __syncthreads();                         // the previous token's reads are done
        for (int i = tid; i < rows; i += kBwdThreads) sx[i] = to_f32(x[((b * L + t) * H + h) * P + p0 + i]);
        for (int i = tid; i < N; i += kBwdThreads) sB[i] = to_f32(Bm[((b * L + t) * G + g) * N + i]);
        __syncthreads();
    };
    auto advance = [&](int64_t t) {              // S <- a_t S + dt_t x_t B_t^T (this CTA's rows)
        stage_xb(t);
        const float dtv = dt[(b * L + t) * H + h];
        const float a = expf(dtv * Ah);
#pragma unroll
        for (int k = 0; k < kMaxPer; ++k) {
            const int e = tid + kBwdThreads * k;
            if (e < E) S[k] = a * S[k] + dtv * sx[e / N] * sB[e % N];
        }
    };

    // forward sweep: checkpoints
    for (int64_t t = 0; t < L; ++t) {
        if (t % kSeg == 0) {
            float* c = ck + (t / kSeg) * (R * N);
#pragma unroll
            for (int k = 0; k < kMaxPer; ++k) {
                const int e = tid + kBwdThreads * k;
                if (e < E) c[e] = S[k];
            }
        }
        advance(t);
    }

    // reverse sweep, one segment at a time
    float dA_acc = 0.f, dD_acc = 0.f;
    for (int64_t s = nseg - 1; s >= 0; --s) {
        const int64_t t0 = s * kSeg, t1 = (t0 + kSeg < L) ? t0 + kSeg : L;
        const float* c = ck + s * (R * N);
#pragma unroll
        for (int k = 0; k < kMaxPer; ++k) {
            const int e = tid + kBwdThreads * k;
            if (e < E) S[k] = c[e];
        }
        for (int64_t t = t0; t < t1; ++t) {
            advance(t);
            if (t + 1 == t1) break;              // S_{t1-1} stays in registers
            float* o = sg + (t - t0) * (R * N);
#pragma unroll
            for (int k = 0; k < kMaxPer; ++k) {
                const int e = tid + kBwdThreads * k;
                if (e < E) o[e] = S[k];
            }
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            __syncthreads();                     // the previous token's reads are done
            for (int i = tid; i < rows; i += kBwdThreads) {
                sx[i] = to_f32(x[((b * L + t) * H + h) * P + p0 + i]);
                sdy[i] = to_f32(dy[((b * L + t) * H + h) * P + p0 + i]);
                rx[i] = 0.f;
            }
            for (int i = tid; i < N; i += kBwdThreads) {
                sB[i] = to_f32(Bm[((b * L + t) * G + g) * N + i]);
                sC[i] = to_f32(Cm[((b * L + t) * G + g) * N + i]);
                rbs[i] = 0.f;
                rcs[i] = 0.f;
            }
            __syncthreads();
            const float dtv = dt[(b * L + t) * H + h];
            const float a = expf(dtv * Ah);
            // S holds S_t (the recompute ended there; each step below moves it
            // back one token); S_{t-1} comes from the segment scratch (this
            // thread's own writes) or the checkpoint
            const float* Sp = (t == t0) ? c : sg + (t - t0 - 1) * (R * N);
            float xgb = 0.f, gs = 0.f;
#pragma unroll
            for (int k = 0; k < kMaxPer; ++k) {
                const int e = tid + kBwdThreads * k;
                if (e < E) {
                    const int pl = e / N, n = e % N;
                    const float gv = Gm[k] + sdy[pl] * sC[n];            // dL/dS_t
                    Gm[k] = gv;
                    const float gb = gv * sB[n];
                    if (warp_rows) {
                        const float r = warp_sum(gb);
                        if (lane == 0) atomicAdd(&rx[pl], r);
                    } else {
                        atomicAdd(&rx[pl], gb);
                    }
                    atomicAdd(&rbs[n], gv * sx[pl]);
                    atomicAdd(&rcs[n], S[k] * sdy[pl]);
                    xgb += sx[pl] * gb;
                    const float sp = Sp[e];
                    gs += gv * sp;
                    S[k] = sp;                                            // S_{t-1}
                }
            }
            xgb = warp_sum(xgb);
            gs = warp_sum(gs);
            if (lane == 0) {
                sw[warp] = xgb;
                sw[4 + warp] = gs;
            }
            __syncthreads();
            for (int i = tid; i < rows; i += kBwdThreads) {
                dx[((b * L + t) * H + h) * P + p0 + i] = Dh * sdy[i] + dtv * rx[i];
                dD_acc += sdy[i] * sx[i];
            }
            for (int i = tid; i < N; i += kBwdThreads) {
                atomicAdd(&dB[((b * L + t) * G + g) * N + i], dtv * rbs[i]);
                atomicAdd(&dC[((b * L + t) * G + g) * N + i], rcs[i]);
            }
            if (tid == 0) {
                float xs = 0.f, gss = 0.f;
                for (int w = 0; w < kBwdThreads / 32; ++w) {
                    xs += sw[w];
                    gss += sw[4 + w];
                }
                atomicAdd(&ddt[(b * L + t) * H + h], xs + Ah * a * gss);
                dA_acc += dtv * a * gss;
            }
#pragma unroll
            for (int k = 0; k < kMaxPer; ++k) Gm[k] *= a;              // dL/dS_{t-1}
        }
    }
    if (dinit) {
#pragma unroll
        for (int k = 0; k < kMaxPer; ++k) {
            const int e = tid + kBwdThreads * k;
            if (e < E) dinit[soff + e] = Gm[k];
        }
    }
    dD_acc = warp_sum(dD_acc);
    __syncthreads();
    if (lane == 0) sw[warp] = dD_acc;
    __syncthreads();
    if (tid == 0) {
        float sum = 0.f;
        for (int w = 0; w < kBwdThreads / 32; ++w) sum += sw[w];
        atomicAdd(&dD[h], sum);
        atomicAdd(&dA[h], dA_acc);
    }
}

int64_t bwd_blocks(const Dims& d) {
    const int R = bwd_rows((int)d.P, (int)d.N);
    return d.b * d.H * (int64_t)((d.P + R - 1) / R);
}

}  // namespace

size_t backward_workspace_bytes(const Dims& d) {
    const int R = bwd_rows((int)d.P, (int)d.N);
    return (size_t)bwd_blocks(d) * (size_t)(bwd_segments(d.L) + kSeg) * (size_t)(R * d.N) * 4;
}

bool backward_supported(const Dims& d) { return d.N <= kElems; }

cudaError_t launch_backward(const void* x, const float* dt, const float* A, const void* B,
                            const void* C, const float* D, const float* init, const void* dy,
                            const float* dfinal, float* dx, float* ddt, float* dA, float* dB,
                            float* dC, float* dD, float* dinit, float* ws, const Dims& d, Elt t,
                            cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(dA, 0, sizeof(float) * (size_t)d.H, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dD, 0, sizeof(float) * (size_t)d.H, s);
    if (e == cudaSuccess && d.b > 0 && d.L > 0) {
        const size_t nbc = sizeof(float) * (size_t)(d.b * d.L * d.G * d.N);
        e = cudaMemsetAsync(dB, 0, nbc, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dC, 0, nbc, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(ddt, 0, sizeof(float) * (size_t)(d.b * d.L * d.H), s);
    }
    if (e != cudaSuccess || d.b == 0) return e;
    if (d.L == 0) {
        // no tokens: the gradient of the initial state is that of the final one
        return dinit ? launch_copy_or_zero(dfinal, dinit, d.b * d.H * d.P * d.N, s) : cudaSuccess;
    }
    const int R = bwd_rows((int)d.P, (int)d.N);
    const size_t smem = sizeof(float) * (size_t)(3 * R + 4 * d.N + 8);
    const dim3 grid((unsigned)bwd_blocks(d));
    if (t == Elt::BF16)
        ssd_bwd_kernel<__nv_bfloat16><<<grid, kBwdThreads, smem, s>>>(
            static_cast<const __nv_bfloat16*>(x), dt, A, static_cast<const __nv_bfloat16*>(B),
            static_cast<const __nv_bfloat16*>(C), D, init, static_cast<const __nv_bfloat16*>(dy),
            dfinal, dx, ddt, dA, dB, dC, dD, dinit, ws, d);
    else
        ssd_bwd_kernel<float><<<grid, kBwdThreads, smem, s>>>(
            static_cast<const float*>(x), dt, A, static_cast<const float*>(B),
            static_cast<const float*>(C), D, init, static_cast<const float*>(dy), dfinal, dx,
            ddt, dA, dB, dC, dD, dinit, ws, d);
    return cudaGetLastError();
}

}  // namespace ssd
