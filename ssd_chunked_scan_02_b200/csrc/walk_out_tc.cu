// walk_out_tc.cu -- the whole tensor-core forward in one launch (bf16, dstate
// 128): walkers (steps a0 + a2 + a3: chunk states and the inter-chunk
// recurrence, state_walk_body.cuh) and output tiles (steps a1 + a4, the
// masked C B^T term, the entering-state term and the skip,
// chunk_out_body.cuh) run side by side, so the output tiles of chunk c start
// as soon as the walkers have written the states entering chunk c instead of
// after the whole walk.
//
// "Transformers are SSMs" (CiteArk), AI research summary: the block
// decomposition (intra-chunk terms as dense contractions, a recurrence over
// chunk states between them); "论文解读：Mamba: ...", 状态空间模型: the
// recurrence taken one chunk per step.
//
// Scheduling.  Every CTA first takes a ticket (one atomic add on a counter
// the host zeroes before the launch).  Tickets 0 .. W-1 are the walkers, one
// per (batch, four heads of one group), each holding an SM to itself;
// tickets W and up are output tiles in chunk-major order.  A walker waits on
// nothing outside its CTA.  An output tile waits (bounded, like every wait
// here) only on walkers, and only for walkers whose tickets were taken before
// its own -- CTAs that are already running -- so the launch makes progress
// whatever order the hardware starts CTAs in and however many fit at once.
// The walker publishes its progress per chunk with a release store after its
// epilogue warps have stored that chunk's entering states and met; the output
// tile's TMA producer acquires it and orders the async proxy behind it before
// loading the entering state.
#include <cuda.h>
#include <cuda_bf16.h>

#include "chunk_out_body.cuh"
#include "common.cuh"
#include "sm100.cuh"
#include "ssd_internal.h"
#include "state_walk_body.cuh"
#include "tc_host.h"
#include "tc_kernels.h"

namespace ssd {
namespace {
using namespace sm100;

constexpr int kHP = 4;                              // heads per walker
constexpr int kThreads = outk::kThreads;
static_assert(walk::Roles<kHP>::kThreads == outk::kThreads, "one block size for both roles");

template <int Q>
struct FusedSmem {
    static constexpr int kWalk = walk::Smem<Q, 128, kHP>::kAlloc;
    static constexpr int kOut = outk::OutSmem<Q, 128>::kAlloc;
    static constexpr int kAlloc = kWalk > kOut ? kWalk : kOut;
    static_assert(kAlloc <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// sched[0]: ticket counter; sched[32 + w]: entering states written by walker w.
template <int Q>
__global__ void __launch_bounds__(kThreads, 1)
walk_out_tc_kernel(const __grid_constant__ CUtensorMap tmXw, const __grid_constant__ CUtensorMap tmBw,
                   const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmH,
                   const __grid_constant__ CUtensorMap tmY, const float* __restrict__ dt,
                   const float* __restrict__ A, const float* __restrict__ Dv,
                   const float* __restrict__ init, __nv_bfloat16* __restrict__ prev,
                   float* __restrict__ fin, int64_t L, int H, int G, int64_t T, int HG,
                   int ksplit, int pcols, int* __restrict__ sched, int nwalk, WaitCtx status) {
    constexpr int kTiles = Q / 128;
    __shared__ int s_ticket;
    if (threadIdx.x == 0) s_ticket = atomicAdd(sched, 1);
    __syncthreads();
    const int tk = s_ticket;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    int* progress = sched + 32;
    const int quads = H >> 2;                       // walkers per batch (H / G a multiple of 4)
    if (tk < nwalk) {
        const int64_t b = tk / quads;
        const int h0 = (tk % quads) * kHP;
        walk::body<Q, 128, kHP>(&tmXw, &tmBw, dt, A, init, prev, fin, L, H, G, T, ksplit, pcols,
                                b, h0 / (H / G), h0, kHP, smem, progress + tk, status);
    } else {
        const int nhg = H / HG;
        const int64_t per_chunk = (int64_t)(nwalk / quads) * kTiles * nhg;   // batch x tiles x groups
        const int64_t o = tk - nwalk;
        const int64_t c = o / per_chunk;
        const int64_t r = o - c * per_chunk;
        const int64_t b = r / (kTiles * nhg);
        const int r2 = (int)(r - b * (kTiles * nhg));
        const int t = r2 / nhg, hg = r2 - t * nhg;
        outk::body<Q, 128>(&tmX, &tmB, &tmC, &tmH, &tmY, dt, A, Dv, L, H, G, T, HG, ksplit, b, c,
                           t, hg * HG, smem, progress, status);
    }
}

template <int Q>
cudaError_t launch_impl(const void* x, const float* dt, const float* A, const void* B,
                        const void* C, const float* D, const float* init, void* prev, void* y,
                        float* fin, int* sched, const Dims& d, int ksplit, int pc, cudaStream_t s) {
    constexpr int N = 128;
    using FS = FusedSmem<Q>;
    CUtensorMap tmXw, tmBw, tmX, tmB, tmC, tmH, tmY;
    // x and y: pc columns a (virtual) head; a 64-column box reads zeros past
    // them and stores only up to them
    const uint64_t xdims[4] = {(uint64_t)pc, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t xstr[3] = {(uint64_t)pc * 2, (uint64_t)(d.H * pc * 2), (uint64_t)(d.L * d.H * pc * 2)};
    const uint64_t bdims[4] = {(uint64_t)N, (uint64_t)d.G, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t bstr[3] = {(uint64_t)N * 2, (uint64_t)(d.G * N * 2), (uint64_t)(d.L * d.G * N * 2)};
    const uint32_t box64[4] = {64, 1, walk::kSub, 1};
    const uint32_t box128[4] = {64, 1, 128, 1};
    cudaError_t e = make_tmap_bf16(&tmXw, x, 4, xdims, xstr, box64);
    if (e == cudaSuccess) e = make_tmap_bf16(&tmBw, B, 4, bdims, bstr, box64);
    if (e == cudaSuccess) e = make_tmap_bf16(&tmX, x, 4, xdims, xstr, box128);
    if (e == cudaSuccess) e = make_tmap_bf16(&tmY, y, 4, xdims, xstr, box128);
    if (e == cudaSuccess) e = make_tmap_bf16(&tmB, B, 4, bdims, bstr, box128);
    if (e == cudaSuccess) e = make_tmap_bf16(&tmC, C, 4, bdims, bstr, box128);
    if (e != cudaSuccess) return e;
    const uint64_t hdims[2] = {(uint64_t)N, (uint64_t)(d.b * d.T * d.H * 64)};
    const uint64_t hstr[1] = {(uint64_t)N * 2};
    const uint32_t hbox[2] = {64, 64};
    e = make_tmap_bf16(&tmH, prev, 2, hdims, hstr, hbox);
    if (e != cudaSuccess) return e;
    const sm100::WaitCtx status = make_wait_ctx();
    if (!status.word) return cudaErrorUnknown;

    const int HG = outk::pick_heads_per_cta(d.H, d.G);
    const int64_t nwalk = d.b * (d.H / kHP);
    const int64_t grid = nwalk + d.b * d.T * (Q / 128) * (d.H / HG);
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    e = cudaMemsetAsync(sched, 0, walk_out_sched_bytes(d), s);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(walk_out_tc_kernel<Q>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             FS::kAlloc);
    if (e != cudaSuccess) return e;
    walk_out_tc_kernel<Q><<<(unsigned)grid, kThreads, FS::kAlloc, s>>>(
        tmXw, tmBw, tmX, tmB, tmC, tmH, tmY, dt, A, D, init, static_cast<__nv_bfloat16*>(prev), fin,
        d.L, (int)d.H, (int)d.G, d.T, HG, ksplit, pc, sched, (int)nwalk, status);
    return cudaGetLastError();
}

}  // namespace

bool walk_out_supported(const Dims& d) {
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    return v.N == 128 && (v.Q == 128 || v.Q == 256) && (v.H / v.G) % kHP == 0 &&
           v.b * (v.H / kHP) <= 0x7fffffffLL;
}

bool walk_out_preferred(const Dims& d) {
    // The overlap pays once the walk is long: with few chunks the output tiles
    // of the last chunk start only when the walk ends, and the two launches
    // (whose walkers, two heads a CTA, walk faster) win (measured: 8 chunks
    // lose, 16 and 32 win).
    return walk_out_supported(d) && d.T >= 16;
}

size_t walk_out_sched_bytes(const Dims& d) {
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    return (size_t)(32 + v.b * (v.H / kHP)) * sizeof(int);
}

cudaError_t launch_walk_out_tc(const void* x, const float* dt, const float* A, const void* B,
                               const void* C, const float* D, const float* init, void* prev,
                               void* y, float* final_states, int* sched, const Dims& d,
                               cudaStream_t s) {
    if (!walk_out_supported(d)) return cudaErrorNotSupported;
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    if (v.Q == 256)
        return launch_impl<256>(x, dt, A, B, C, D, init, prev, y, final_states, sched, v, k,
                                head_cols(d), s);
    return launch_impl<128>(x, dt, A, B, C, D, init, prev, y, final_states, sched, v, k,
                            head_cols(d), s);
}

}  // namespace ssd
