// state_pass.cu -- the sequential inter-chunk state recurrence (step 3 of the
// block-decomposed SSD forward), in fp32:
//     h_{-1} = init (or 0),   prev_c = h_{c-1},   h_c = exp(logdecay_c) h_{c-1} + S_c
// where S_c is the chunk's own state (chunk started from zero) and logdecay_c
// = sum_{t in chunk c} dt_t A_h.  The backward runs the same recurrence with
// the chunks in reverse order: g_{T-1} = dL/dfinal, out_c = g_c (dL/dh of the
// state chunk c hands on), g_{c-1} = exp(logdecay_c) g_c + dS_c, dL/dinit =
// g_{-1}.  "论文解读：Mamba: ...", 状态空间模型: the
// linear-recurrence form, here taken one chunk per step instead of one token.
//
// Every (batch, head, p, n) state element is an independent chain; a thread
// owns VEC consecutive elements (16-byte fp32 loads), walks the chunks in
// order and keeps the chain in registers.  Loads of later chunks do not
// depend on the chain: a register ring keeps 16 chunks' loads in flight, so
// the walk stays bandwidth-bound even with few chains (one long sequence).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kAhead = 16;   // chunks whose loads are in flight per thread

template <typename TP, int VEC>
struct Store;
template <typename TP, int VEC>
struct StoreLo {
    static __device__ __forceinline__ void run(TP*, const float*) {}
};
template <int VEC>
struct Store<float, VEC> {
    static __device__ __forceinline__ void run(float* dst, const float* v) {
        if constexpr (VEC == 4) {
            *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
#pragma unroll
            for (int k = 0; k < VEC; ++k) dst[k] = v[k];
        }
    }
};
template <int VEC>
struct Store<__nv_bfloat16, VEC> {
    static __device__ __forceinline__ void run(__nv_bfloat16* dst, const float* v) {
        if constexpr (VEC == 4) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]);
            __nv_bfloat162 hi = __floats2bfloat162_rn(v[2], v[3]);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t*>(&lo);
            u.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(dst) = u;
        } else {
#pragma unroll
            for (int k = 0; k < VEC; ++k) dst[k] = __float2bfloat16_rn(v[k]);
        }
    }
};

template <int VEC>
__device__ __forceinline__ void load_vec(const float* __restrict__ src, float* v) {
    if constexpr (VEC == 4) {
        const float4 q = *reinterpret_cast<const float4*>(src);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
        for (int k = 0; k < VEC; ++k) v[k] = src[k];
    }
}

// The rounding residue of a bf16 store: lo = bf16(v - bf16(v)), so that
// hi + lo carries v to about 16 bits more than hi alone.
template <int VEC>
struct StoreLo<__nv_bfloat16, VEC> {
    static __device__ __forceinline__ void run(__nv_bfloat16* dst, const float* v) {
        float r[VEC];
#pragma unroll
        for (int k = 0; k < VEC; ++k) r[k] = v[k] - __bfloat162float(__float2bfloat16_rn(v[k]));
        Store<__nv_bfloat16, VEC>::run(dst, r);
    }
};

template <typename TP, int VEC>
__global__ void __launch_bounds__(256)
state_pass_kernel(const float* __restrict__ states, const float* __restrict__ logdecay,
                  const float* __restrict__ init, TP* __restrict__ prev,
                  float* __restrict__ fin, int64_t b, int64_t T, int64_t H, int64_t PN,
                  int reverse, int64_t N, int64_t p_ext, TP* __restrict__ prev_lo) {
    const int64_t nvec = PN / VEC;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= b * H * nvec) return;
    const int64_t bh = idx / nvec;
    const int64_t off = (idx - bh * nvec) * VEC;
    const int64_t bb = bh / H, h = bh - bb * H;

    // init and fin: (b, H, p_ext, N) when p_ext rows of the PN / N are the caller's
    const int64_t p = off / N;
    const bool ext_row = p < p_ext;
    const int64_t ext = (bh * p_ext + p) * N + (off - p * N);
    float hs[VEC];
    if (init && ext_row) {
        load_vec<VEC>(init + ext, hs);
    } else {
#pragma unroll
        for (int k = 0; k < VEC; ++k) hs[k] = 0.f;
    }
    // chunk order: 0 .. T-1, or T-1 .. 0 (reverse)
    const int64_t c_first = reverse ? T - 1 : 0;
    const int64_t cstride = reverse ? -H * PN : H * PN;
    const int64_t lstride = reverse ? -H : H;
    const float* sp = states + ((bb * T + c_first) * H + h) * PN + off;
    const float* lp = logdecay + (bb * T + c_first) * H + h;
    TP* pp = prev + ((bb * T + c_first) * H + h) * PN + off;
    TP* pl = prev_lo ? prev_lo + ((bb * T + c_first) * H + h) * PN + off : nullptr;
    // a ring of kAhead chunks' states and log-decays in registers: the loads
    // of chunk c + kAhead are issued when chunk c is consumed
    float sv[kAhead][VEC], lv[kAhead];
    const float* sq = sp;                    // the next chunk to load
    const float* lq = lp;
    int64_t cl = 0;
#pragma unroll
    for (int k = 0; k < kAhead; ++k) {
        if (cl < T) {
            load_vec<VEC>(sq, sv[k]);
            lv[k] = *lq;
        }
        sq += cstride;
        lq += lstride;
        ++cl;
    }
    TP* pq = pp;
    for (int64_t c0 = 0; c0 < T; c0 += kAhead) {
#pragma unroll
        for (int k = 0; k < kAhead; ++k) {
            if (c0 + k >= T) break;
            const float a = expf(lv[k]);
            Store<TP, VEC>::run(pq, hs);
            pq += cstride;
            if (pl) {
                StoreLo<TP, VEC>::run(pl, hs);
                pl += cstride;
            }
#pragma unroll
            for (int e = 0; e < VEC; ++e) hs[e] = fmaf(a, hs[e], sv[k][e]);
            if (cl < T) {
                load_vec<VEC>(sq, sv[k]);
                lv[k] = *lq;
            }
            sq += cstride;
            lq += lstride;
            ++cl;
        }
    }
    if (fin && ext_row) {
        float* fp = fin + ext;
#pragma unroll
        for (int k = 0; k < VEC; ++k) fp[k] = hs[k];
    }
}

__global__ void copy_or_zero_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                    int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) dst[i] = src ? src[i] : 0.f;
}

template <typename TP, int VEC>
cudaError_t run(const float* states, const float* logdecay, const float* init, void* prev,
                float* fin, const Dims& d, bool reverse, int64_t p_ext, void* prev_lo, cudaStream_t s) {
    const int64_t PN = d.P * d.N;
    const int64_t threads = d.b * d.H * (PN / VEC);
    if (threads == 0) return cudaSuccess;
    const int bs = 256;
    const int64_t blocks = (threads + bs - 1) / bs;
    state_pass_kernel<TP, VEC><<<(unsigned)blocks, bs, 0, s>>>(
        states, logdecay, init, static_cast<TP*>(prev), fin, d.b, d.T, d.H, PN, reverse ? 1 : 0,
        d.N, p_ext, static_cast<TP*>(prev_lo));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_pass(const float* states, const float* logdecay, const float* init,
                              void* prev, float* fin, const Dims& d, Elt t, cudaStream_t s,
                              bool reverse, int64_t p_ext, void* prev_lo) {
    // with p_ext rows a vector of 4 must stay within one state row
    const int64_t pe = (p_ext > 0 && p_ext < d.P) ? p_ext : d.P;
    const bool v4 = pe == d.P ? ((d.P * d.N) % 4) == 0 : (d.N % 4) == 0;
    if (t == Elt::F32)
        return v4 ? run<float, 4>(states, logdecay, init, prev, fin, d, reverse, pe, nullptr, s)
                  : run<float, 1>(states, logdecay, init, prev, fin, d, reverse, pe, nullptr, s);
    return v4 ? run<__nv_bfloat16, 4>(states, logdecay, init, prev, fin, d, reverse, pe, prev_lo, s)
              : run<__nv_bfloat16, 1>(states, logdecay, init, prev, fin, d, reverse, pe, prev_lo, s);
}

cudaError_t launch_copy_or_zero(const float* init, float* fin, int64_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    copy_or_zero_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(init, fin, n);
    return cudaGetLastError();
}

}  // namespace ssd
