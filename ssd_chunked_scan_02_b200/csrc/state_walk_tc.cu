// state_walk_tc.cu -- the standalone walk kernel: chunk states and the
// inter-chunk recurrence in one pass (steps a0 + a2 + a3 of the
// block-decomposed SSD forward, bf16 inputs), one CTA per (batch, head pair
// of one group) walking the chunks in order (the walker is in
// state_walk_body.cuh).  Heads are the kernels' virtual heads of headdim 64
// (a head of headdim 64 k is k of them); a group with an odd number of heads
// pairs its last head with a zero phantom.  Sized for two CTAs per SM (about
// 105 KB of shared memory and 256 or 128 TMEM columns each).
//
// "论文解读：Mamba: ...", 状态空间模型: the linear-recurrence form, taken one
// chunk per step; "Transformers are SSMs" (CiteArk), AI research summary: the
// chunk's contribution is one dense contraction.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"
#include "ssd_internal.h"
#include "state_walk_body.cuh"
#include "tc_host.h"
#include "tc_kernels.h"

namespace ssd {
namespace {
using namespace sm100;

constexpr int kThreads = walk::Roles<2>::kThreads;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int Q, int N>
__global__ void __launch_bounds__(kThreads, 2)
state_walk_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                     const float* __restrict__ dt, const float* __restrict__ A,
                     const float* __restrict__ init, __nv_bfloat16* __restrict__ prev,
                     float* __restrict__ fin, int64_t L, int H, int G, int64_t T,
                     int ksplit, int pcols, WaitCtx status) {
    const HeadPairs hp(H, G);
    const int64_t b = blockIdx.x / (G * hp.per_group());
    int g, h0;
    bool has1;
    hp.map((int)(blockIdx.x % (G * hp.per_group())), &g, &h0, &has1);
    extern __shared__ uint8_t smem_raw[];
    walk::body<Q, N, 2>(&tmX, &tmB, dt, A, init, prev, fin, L, H, G, T, ksplit, pcols, b, g, h0,
                        has1 ? 2 : 1, align1024(smem_raw), nullptr, status);
}

template <int Q, int N>
cudaError_t launch_impl(const void* x, const float* dt, const float* A, const void* B,
                        const float* init, void* prev, float* fin, const Dims& d, int ksplit,
                        int pc, cudaStream_t s) {
    using S = walk::Smem<Q, N, 2>;
    CUtensorMap tmX, tmB;
    // x: pc columns a (virtual) head; a 64-column box reads zeros past them
    const uint64_t xdims[4] = {(uint64_t)pc, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t xstr[3] = {(uint64_t)pc * 2, (uint64_t)(d.H * pc * 2), (uint64_t)(d.L * d.H * pc * 2)};
    const uint32_t box[4] = {64, 1, walk::kSub, 1};
    cudaError_t e = make_tmap_bf16(&tmX, x, 4, xdims, xstr, box);
    if (e != cudaSuccess) return e;
    const uint64_t bdims[4] = {(uint64_t)N, (uint64_t)d.G, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t bstr[3] = {(uint64_t)N * 2, (uint64_t)(d.G * N * 2), (uint64_t)(d.L * d.G * N * 2)};
    e = make_tmap_bf16(&tmB, B, 4, bdims, bstr, box);
    if (e != cudaSuccess) return e;
    const sm100::WaitCtx status = make_wait_ctx();
    if (!status.word) return cudaErrorUnknown;
    e = cudaFuncSetAttribute(state_walk_tc_kernel<Q, N>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
    if (e != cudaSuccess) return e;
    const int64_t grid = d.b * d.G * HeadPairs((int)d.H, (int)d.G).per_group();
    state_walk_tc_kernel<Q, N><<<(unsigned)grid, kThreads, S::kAlloc, s>>>(
        tmX, tmB, dt, A, init, static_cast<__nv_bfloat16*>(prev), fin, d.L, (int)d.H, (int)d.G,
        d.T, ksplit, pc, status);
    return cudaGetLastError();
}

}  // namespace

bool walk_preferred(const Dims& d) {
    // One walker per (batch, head pair), each progressing chunk by chunk:
    // the walk pays off once there are enough walkers to keep most SMs busy
    // (measured: 96 walkers and more beat chunk states + state pass at every
    // workload shape, 64 and fewer lose to them).
    int ksplit = 1;
    const Dims v = virtual_heads(d, &ksplit);
    const int64_t walkers = v.b * v.G * HeadPairs((int)v.H, (int)v.G).per_group();
    return walkers >= 96 && walkers <= 0x7fffffffLL;
}

cudaError_t launch_state_walk_tc(const void* x, const float* dt, const float* A, const void* B,
                                 const float* init, void* prev, float* fin, const Dims& d,
                                 cudaStream_t s) {
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    if (v.b * v.G * HeadPairs((int)v.H, (int)v.G).per_group() > 0x7fffffffLL)
        return cudaErrorInvalidValue;
    if (v.Q == 256 && v.N == 128) return launch_impl<256, 128>(x, dt, A, B, init, prev, fin, v, k, head_cols(d), s);
    if (v.Q == 256 && v.N == 64) return launch_impl<256, 64>(x, dt, A, B, init, prev, fin, v, k, head_cols(d), s);
    if (v.Q == 128 && v.N == 128) return launch_impl<128, 128>(x, dt, A, B, init, prev, fin, v, k, head_cols(d), s);
    if (v.Q == 128 && v.N == 64) return launch_impl<128, 64>(x, dt, A, B, init, prev, fin, v, k, head_cols(d), s);
    return cudaErrorNotSupported;
}

}  // namespace ssd
