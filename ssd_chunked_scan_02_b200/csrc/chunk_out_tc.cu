// chunk_out_tc.cu -- the output kernel: chunk outputs on the tcgen05 tensor
// cores (steps a1 + a4 of the block-decomposed SSD forward, bf16 inputs),
// one CTA per (batch, chunk, 128-row tile, group of heads sharing B and C);
// the tile's work is in chunk_out_body.cuh.
//
// "Transformers are SSMs" (CiteArk), what this means: the 1-semiseparable SSM
// restricted to a chunk is structured masked attention, C B^T masked by the
// decay; review page, 核心概念 items 3 and 5; 关键洞察 item 1.
#include <cuda.h>
#include <cuda_bf16.h>

#include "chunk_out_body.cuh"
#include "common.cuh"
#include "sm100.cuh"
#include "ssd_internal.h"
#include "tc_host.h"
#include "tc_kernels.h"

namespace ssd {
namespace {
using namespace sm100;
using outk::kThreads;
using outk::kMaxHeads;
using outk::OutSmem;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int Q, int N>
__global__ void __launch_bounds__(kThreads, 1)
chunk_out_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmH,
                    const __grid_constant__ CUtensorMap tmY, const float* __restrict__ dt,
                    const float* __restrict__ A, const float* __restrict__ Dv, int64_t L, int H,
                    int G, int64_t T, int HG, int ksplit, WaitCtx status) {
    constexpr int kTiles = Q / 128;
    const int64_t bx = blockIdx.x;
    const int t = (int)(bx % kTiles);
    const int64_t bt = bx / kTiles;
    extern __shared__ uint8_t smem_raw[];
    outk::body<Q, N>(&tmX, &tmB, &tmC, &tmH, &tmY, dt, A, Dv, L, H, G, T, HG, ksplit, bt / T,
                     bt % T, t, (int)blockIdx.y * HG, align1024(smem_raw), nullptr, 1, true, status);
}

template <int Q, int N>
cudaError_t launch_impl(const void* x, const float* dt, const float* A, const void* B,
                        const void* C, const float* D, const void* prev, void* y, const Dims& d, int ksplit,
                        int pc, cudaStream_t s) {
    using S = OutSmem<Q, N>;
    CUtensorMap tmX, tmB, tmC, tmH, tmY;
    // x and y: pc columns a (virtual) head; a 64-column box reads zeros past
    // them and stores only up to them
    const uint64_t xdims[4] = {(uint64_t)pc, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t xstr[3] = {(uint64_t)pc * 2, (uint64_t)(d.H * pc * 2), (uint64_t)(d.L * d.H * pc * 2)};
    const uint32_t box128[4] = {64, 1, 128, 1};
    cudaError_t e = make_tmap_bf16(&tmX, x, 4, xdims, xstr, box128);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&tmY, y, 4, xdims, xstr, box128);
    if (e != cudaSuccess) return e;
    const uint64_t bdims[4] = {(uint64_t)N, (uint64_t)d.G, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t bstr[3] = {(uint64_t)N * 2, (uint64_t)(d.G * N * 2),
                              (uint64_t)(d.L * d.G * N * 2)};
    e = make_tmap_bf16(&tmB, B, 4, bdims, bstr, box128);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&tmC, C, 4, bdims, bstr, box128);
    if (e != cudaSuccess) return e;
    const uint64_t hdims[2] = {(uint64_t)N, (uint64_t)(d.b * d.T * d.H * 64)};
    const uint64_t hstr[1] = {(uint64_t)N * 2};
    const uint32_t hbox[2] = {64, 64};
    e = make_tmap_bf16(&tmH, prev, 2, hdims, hstr, hbox);
    if (e != cudaSuccess) return e;
    const sm100::WaitCtx status = make_wait_ctx();
    if (!status.word) return cudaErrorUnknown;

    const int HG = outk::pick_heads_per_cta(d.H, d.G);
    e = cudaFuncSetAttribute(chunk_out_tc_kernel<Q, N>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(d.b * d.T * (Q / 128)), (unsigned)(d.H / HG));
    chunk_out_tc_kernel<Q, N><<<grid, kThreads, S::kAlloc, s>>>(
        tmX, tmB, tmC, tmH, tmY, dt, A, D, d.L, (int)d.H,
        (int)d.G, d.T, HG, ksplit, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_out_tc(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, const void* prev, void* y,
                                const Dims& d, cudaStream_t s) {
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    if (v.Q == 256 && v.N == 128) return launch_impl<256, 128>(x, dt, A, B, C, D, prev, y, v, k, head_cols(d), s);
    if (v.Q == 256 && v.N == 64) return launch_impl<256, 64>(x, dt, A, B, C, D, prev, y, v, k, head_cols(d), s);
    if (v.Q == 128 && v.N == 128) return launch_impl<128, 128>(x, dt, A, B, C, D, prev, y, v, k, head_cols(d), s);
    if (v.Q == 128 && v.N == 64) return launch_impl<128, 64>(x, dt, A, B, C, D, prev, y, v, k, head_cols(d), s);
    return cudaErrorNotSupported;
}

}  // namespace ssd
