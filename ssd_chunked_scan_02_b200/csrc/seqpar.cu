// seqpar.cu -- the pieces of the sequence-parallel forward (a sequence split
// into shards along L, one per rank, with one exchange):
//
//   ssd_seq_logdecay            Lambda[b,h] = sum_t dt[b,t,h] A[h]            (per shard)
//   ssd_state_exchange_combine  h_0 = init, h_{q+1} = exp(Lambda_q) h_q + F_q  (rank order)
//   ssd_state_correction_fwd    y_t += exp(cs_t) h_in C_t,  final += exp(cs_last) h_in
//
// "Transformers are SSMs" (CiteArk), what this means: the layer suits
// large-scale (model-parallel) training.  The state entering a shard acts on
// the shard linearly, which is what lets each rank run its shard from a zero
// state and fix its outputs up afterwards.
//
// The correction needs cs_t, the running sum of dt*A from the shard's first
// token.  A prep kernel (one CTA per (batch, head)) sums dt*A over every
// 128-token tile in fp64 and writes each tile's exclusive prefix (log2
// units, fp32), so that the correction's CTAs, one per (batch, tile, head
// block), start from their tile's offset independently; it also advances the
// final state by exp(Lambda) h_in and, for the tensor-core path, writes h_in
// rounded to bf16 (the MMA operand).  Tiles whose decay has underflowed to
// zero (A <= 0) skip their work: their correction is exactly zero.
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "seqpar.h"

namespace ssd {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTile = kSeqparTile;      // tokens per correction tile

// ------------------------------------------------------------------ log-decay of a shard
// CTA per (batch, head): 256 threads, each summing every 256th token with four
// independent fp64 partial sums, then a block reduction.
__global__ void __launch_bounds__(256)
seq_logdecay_kernel(const float* __restrict__ dt, const float* __restrict__ A,
                    float* __restrict__ out, int64_t L, int H) {
    const int64_t b = blockIdx.x / H;
    const int h = (int)(blockIdx.x % H);
    const int tid = threadIdx.x;
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    const float* p = dt + b * L * H + h;
    int64_t t = tid;
    for (; t + 768 < L; t += 1024) {
        s0 += (double)p[t * H];
        s1 += (double)p[(t + 256) * H];
        s2 += (double)p[(t + 512) * H];
        s3 += (double)p[(t + 768) * H];
    }
    for (; t < L; t += 256) s0 += (double)p[t * H];
    double s = (s0 + s1) + (s2 + s3);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    __shared__ double part[8];
    if ((tid & 31) == 0) part[tid >> 5] = s;
    __syncthreads();
    if (tid == 0) {
        double tot = 0.0;
        for (int w = 0; w < 8; ++w) tot += part[w];
        out[b * H + h] = (float)(tot * (double)A[h]);
    }
}

// ------------------------------------------------------------------ exchange combine
// Thread per VEC consecutive state elements of one (batch, head): the fold
// over the ranks before `rank`, one decay factor per rank.
template <int VEC>
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ F, const float* __restrict__ ld,
               const float* __restrict__ init, float* __restrict__ out, int rank, int64_t BH,
               int64_t PN) {
    const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * VEC;
    if (i >= BH * PN) return;
    const int64_t bh = i / PN;
    float h[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) h[e] = init ? init[i + e] : 0.f;
    for (int q = 0; q < rank; ++q) {
        const float a = expf(ld[(int64_t)q * BH + bh]);
        const float* f = F + (int64_t)q * BH * PN + i;
        if constexpr (VEC == 4) {
            const float4 v = *reinterpret_cast<const float4*>(f);
            h[0] = fmaf(a, h[0], v.x); h[1] = fmaf(a, h[1], v.y);
            h[2] = fmaf(a, h[2], v.z); h[3] = fmaf(a, h[3], v.w);
        } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) h[e] = fmaf(a, h[e], f[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) out[i + e] = h[e];
}

// ------------------------------------------------------------------ correction prep
// CTA per (batch, head): tile prefixes (log2 units), final += exp(Lambda) h_in,
// optionally h_in -> bf16.
__global__ void __launch_bounds__(256)
correction_prep_kernel(const float* __restrict__ h_in, const float* __restrict__ dt,
                       const float* __restrict__ A, float* __restrict__ tile_prefix,
                       float* __restrict__ fin, __nv_bfloat16* __restrict__ h_bf16, int64_t L,
                       int H, int64_t ntiles, int64_t PN) {
    const int64_t b = blockIdx.x / H;
    const int h = (int)(blockIdx.x % H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kBatch = 1024;
    __shared__ double tsum[kBatch];
    __shared__ double s_carry;
    if (tid == 0) s_carry = 0.0;
    const double Ah = (double)A[h] * (double)kLog2e;
    for (int64_t k0 = 0; k0 < ntiles; k0 += kBatch) {
        const int nk = (int)((ntiles - k0) < kBatch ? (ntiles - k0) : kBatch);
        for (int k = warp; k < nk; k += 8) {
            const int64_t t0 = (k0 + k) * kTile;
            float v[kTile / 32];
#pragma unroll
            for (int j = 0; j < kTile / 32; ++j) {
                const int64_t t = t0 + lane + 32 * j;
                v[j] = (t < L) ? dt[(b * L + t) * H + h] : 0.f;
            }
            double s = 0.0;
#pragma unroll
            for (int j = 0; j < kTile / 32; ++j) s += (double)v[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) tsum[k] = s * Ah;
        }
        __syncthreads();
        if (tid == 0) {
            double c = s_carry;
            for (int k = 0; k < nk; ++k) {
                tile_prefix[(b * ntiles + k0 + k) * H + h] = (float)c;
                c += tsum[k];
            }
            s_carry = c;
        }
        __syncthreads();
    }
    const float decay = exp2f((float)s_carry);          // exp(Lambda): the whole shard
    const float* hp = h_in + (b * H + h) * PN;
    for (int64_t i = tid; i < PN; i += 256) {
        const float v = hp[i];
        if (fin) fin[(b * H + h) * PN + i] = fmaf(decay, v, fin[(b * H + h) * PN + i]);
        if (h_bf16) h_bf16[(b * H + h) * PN + i] = __float2bfloat16_rn(v);
    }
}

// ------------------------------------------------------------------ exact correction (SIMT)
// CTA per (batch, 128-token tile, head, block of PB state rows): y rows of the
// tile += alpha_t (h_in[p, :] . C_t), alpha_t = 2^(prefix + cs_t); fp32 FMAs.
template <typename TX>
__global__ void __launch_bounds__(256)
correction_simt_kernel(const float* __restrict__ h_in, const float* __restrict__ dt,
                       const float* __restrict__ A, const TX* __restrict__ C,
                       const float* __restrict__ tile_prefix, TX* __restrict__ y, int64_t L,
                       int H, int G, int P, int N, int PB, int64_t ntiles) {
    extern __shared__ float sm[];
    const int tid = threadIdx.x;
    const int64_t bk = blockIdx.x;
    const int64_t k = bk % ntiles, b = bk / ntiles;
    const int h = blockIdx.y;
    const int p0 = blockIdx.z * PB;
    const int np = (P - p0) < PB ? (P - p0) : PB;
    const int g = h / (H / G);
    const int64_t t0 = k * kTile;
    const int len = (int)((L - t0) < kTile ? (L - t0) : kTile);
    const float Ah = A[h] * kLog2e;
    const float pre = tile_prefix[(b * ntiles + k) * H + h];
    // a decay that has underflowed stays zero for a non-growing state
    if (Ah <= 0.f && exp2f(pre) == 0.f) return;

    float* s_alpha = sm;                        // [kTile]
    float* s_h = s_alpha + kTile;               // [PB][N + 1]
    float* s_c = s_h + PB * (N + 1);            // [32][N + 1]
    // alpha_t: inclusive scan of dt*A (log2) over the tile, by warps 0-3
    __shared__ float s_ws[4];
    if (tid < kTile) {
        float v = (tid < len) ? dt[(b * L + t0 + tid) * H + h] * Ah : 0.f;
        const int lane = tid & 31;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        if (lane == 31) s_ws[tid >> 5] = v;
        s_alpha[tid] = v;
    }
    for (int i = tid; i < np * N; i += 256) {
        const int r = i / N, n = i - r * N;
        s_h[r * (N + 1) + n] = h_in[((b * H + h) * P + p0 + r) * (int64_t)N + n];
    }
    __syncthreads();
    if (tid < kTile) {
        float off = 0.f;
        for (int w = 0; w < (tid >> 5); ++w) off += s_ws[w];
        s_alpha[tid] = exp2f(pre + s_alpha[tid] + off);
    }
    // 32-token sub-tiles: thread (token pair tt, p group pg) computes 2 x (PB/16) outputs
    // (PB <= 64)
    const int tt = tid >> 4, pg = tid & 15;
    for (int s0 = 0; s0 < len; s0 += 32) {
        __syncthreads();                        // s_c free; s_alpha published
        for (int i = tid; i < 32 * N; i += 256) {
            const int r = i / N, n = i - r * N;
            const int64_t t = t0 + s0 + r;
            s_c[r * (N + 1) + n] = (s0 + r < len) ? to_f32(C[((b * L + t) * G + g) * (int64_t)N + n]) : 0.f;
        }
        __syncthreads();
        float acc[2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
        const float* c0 = s_c + (2 * tt) * (N + 1);
        const float* c1 = c0 + (N + 1);
        for (int n = 0; n < N; ++n) {
            const float ca = c0[n], cb = c1[n];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = pg + 16 * q;
                if (r < np) {
                    const float hv = s_h[r * (N + 1) + n];
                    acc[0][q] = fmaf(hv, ca, acc[0][q]);
                    acc[1][q] = fmaf(hv, cb, acc[1][q]);
                }
            }
        }
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            const int j = s0 + 2 * tt + a;
            if (j >= len) continue;
            const float al = s_alpha[j];
            TX* yr = y + ((b * L + t0 + j) * H + h) * (int64_t)P + p0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = pg + 16 * q;
                if (r < np) yr[r] = from_f32<TX>(fmaf(al, acc[a][q], to_f32(yr[r])));
            }
        }
    }
}

}  // namespace

cudaError_t launch_seq_logdecay(const float* dt, const float* A, float* out, const Dims& d,
                                cudaStream_t s) {
    if (d.b * d.H == 0) return cudaSuccess;
    seq_logdecay_kernel<<<(unsigned)(d.b * d.H), 256, 0, s>>>(dt, A, out, d.L, (int)d.H);
    return cudaGetLastError();
}

cudaError_t launch_state_combine(const float* F, const float* ld, const float* init, float* out,
                                 int rank, const Dims& d, cudaStream_t s) {
    const int64_t BH = d.b * d.H, PN = d.P * d.N;
    if (BH * PN == 0) return cudaSuccess;
    if (PN % 4 == 0) {
        const int64_t n = BH * PN / 4;
        combine_kernel<4><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(F, ld, init, out, rank, BH, PN);
    } else {
        combine_kernel<1><<<(unsigned)((BH * PN + 255) / 256), 256, 0, s>>>(F, ld, init, out, rank,
                                                                            BH, PN);
    }
    return cudaGetLastError();
}

int64_t correction_tiles(const Dims& d) { return (d.L + kTile - 1) / kTile; }

cudaError_t launch_correction_prep(const float* h_in, const float* dt, const float* A,
                                   float* tile_prefix, float* fin, __nv_bfloat16* h_bf16,
                                   const Dims& d, cudaStream_t s) {
    if (d.b * d.H == 0) return cudaSuccess;
    correction_prep_kernel<<<(unsigned)(d.b * d.H), 256, 0, s>>>(
        h_in, dt, A, tile_prefix, fin, h_bf16, d.L, (int)d.H, correction_tiles(d), d.P * d.N);
    return cudaGetLastError();
}

cudaError_t launch_correction_simt(const float* h_in, const float* dt, const float* A,
                                   const void* C, const float* tile_prefix, void* y,
                                   const Dims& d, Elt t, cudaStream_t s) {
    const int64_t nt = correction_tiles(d);
    if (d.b * nt == 0) return cudaSuccess;
    const int PB = (int)(d.P < 64 ? d.P : 64);
    const size_t smem = (size_t)(kTile + PB * (d.N + 1) + 32 * (d.N + 1)) * 4;
    dim3 grid((unsigned)(d.b * nt), (unsigned)d.H, (unsigned)((d.P + PB - 1) / PB));
    if (t == Elt::F32) {
        cudaError_t e = cudaFuncSetAttribute(correction_simt_kernel<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        correction_simt_kernel<float><<<grid, 256, smem, s>>>(
            h_in, dt, A, static_cast<const float*>(C), tile_prefix, static_cast<float*>(y), d.L,
            (int)d.H, (int)d.G, (int)d.P, (int)d.N, PB, nt);
    } else {
        cudaError_t e = cudaFuncSetAttribute(correction_simt_kernel<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        correction_simt_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(
            h_in, dt, A, static_cast<const __nv_bfloat16*>(C), tile_prefix,
            static_cast<__nv_bfloat16*>(y), d.L, (int)d.H, (int)d.G, (int)d.P, (int)d.N, PB, nt);
    }
    return cudaGetLastError();
}

}  // namespace ssd
