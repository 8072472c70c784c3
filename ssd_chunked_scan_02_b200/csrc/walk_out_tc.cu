// walk_out_tc.cu -- the whole tensor-core forward in one launch (bf16):
// walkers (steps a0 + a2 + a3: chunk states and the inter-chunk
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
// per (batch, HP heads of one group: four for dstate 128, two for dstate
// 64), each holding an SM to itself;
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

constexpr int kThreads = outk::kThreads;
static_assert(walk::Roles<4>::kThreads <= outk::kThreads, "one block size for both roles");
static_assert(walk::Roles<2>::kThreads <= outk::kThreads, "one block size for both roles");

template <int Q, int N, int HP>
struct FusedSmem {
    static constexpr int kWalk = walk::Smem<Q, N, HP>::kAlloc;
    static constexpr int kOut = outk::OutSmem<Q, N>::kAlloc;
    static constexpr int kAlloc = kWalk > kOut ? kWalk : kOut;
    static_assert(kAlloc <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// The launch's shape: HP heads a walker, HG heads an output tile (HG2 in the
// last KS chunks: smaller tiles there shorten the launch's ragged end).
struct Cfg {
    int hp, hg, hg2, ks;
};

Cfg config(const Dims& v) {
    Cfg c;
    // walkers of two heads walk faster (4.5 against 6 us a chunk) but take
    // twice the SMs from the output tiles; with dstate 128 (a walker of four
    // heads fits TMEM) four heads come out ahead at every measured size
    c.hp = (v.N == 128) ? 4 : 2;
    c.hg = outk::pick_heads_per_cta(v.H, v.G);
    // enough output tiles to spread over the SMs: halve the heads a tile
    // while the launch has fewer than 256 tiles
    while (c.hg % 2 == 0 && c.hg >= 8 && v.b * v.T * (v.Q / 128) * (v.H / c.hg) < 256)
        c.hg /= 2;
    c.ks = (c.hg % 2 == 0 && c.hg >= 8 && v.T > 2) ? 2 : 0;
    c.hg2 = c.ks ? c.hg / 2 : c.hg;
    return c;
}

// Output tiles of chunks [0, T - ks) (hg heads each) then of the last ks
// chunks (hg2 heads each), each chunk's in (batch, row block, head block)
// order.
int64_t out_tiles(const Dims& v, const Cfg& c) {
    const int64_t per = v.b * (v.Q / 128);
    return per * ((v.T - c.ks) * (v.H / c.hg) + c.ks * (v.H / c.hg2));
}

int64_t walkers(const Dims& v, int hp) {
    const int64_t hpg = v.H / v.G;
    return v.b * v.G * ((hpg + hp - 1) / hp);
}

// sched[0]: ticket counter; sched[32 + w]: entering states written by walker w.
template <int Q, int N, int HP>
__global__ void __launch_bounds__(kThreads, 1)
walk_out_tc_kernel(const __grid_constant__ CUtensorMap tmXw, const __grid_constant__ CUtensorMap tmBw,
                   const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmH,
                   const __grid_constant__ CUtensorMap tmY, const float* __restrict__ dt,
                   const float* __restrict__ A, const float* __restrict__ Dv,
                   const float* __restrict__ init, __nv_bfloat16* __restrict__ prev,
                   float* __restrict__ fin, int64_t L, int H, int G, int64_t T, int HG,
                   int HG2, int KS, int ksplit, int pcols, int* __restrict__ sched, int nwalk,
                   WaitCtx status) {
    constexpr int kTiles = Q / 128;
    __shared__ int s_ticket;
    if (threadIdx.x == 0) s_ticket = atomicAdd(sched, 1);
    __syncthreads();
    const int tk = s_ticket;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    int* progress = sched + 32;
    const int hpg = H / G;
    const int wpg = (hpg + HP - 1) / HP;             // walkers a group
    if (tk < nwalk) {
        const int64_t b = tk / (G * wpg);
        const int r = tk % (G * wpg);
        const int g = r / wpg, l = r % wpg;
        const int h0 = g * hpg + HP * l;
        const int nreal = hpg - HP * l < HP ? hpg - HP * l : HP;
        walk::body<Q, N, HP>(&tmXw, &tmBw, dt, A, init, prev, fin, L, H, G, T, ksplit, pcols,
                             b, g, h0, nreal, smem, progress + tk, status);
    } else {
        const int64_t nb = nwalk / (G * wpg);           // batch
        const int64_t first = (T - KS) * nb * kTiles * (H / HG);
        int64_t o = tk - nwalk;
        int hgs = HG;
        int64_t c0 = 0;
        if (o >= first) {                               // the last KS chunks: smaller tiles
            o -= first;
            hgs = HG2;
            c0 = T - KS;
        }
        const int nhg = H / hgs;
        const int64_t per_chunk = nb * kTiles * nhg;    // batch x row blocks x head blocks
        const int64_t c = c0 + o / per_chunk;
        const int64_t r = o % per_chunk;
        const int64_t b = r / (kTiles * nhg);
        const int r2 = (int)(r - b * (kTiles * nhg));
        const int t = r2 / nhg, hg = r2 - t * nhg;
        outk::body<Q, N>(&tmX, &tmB, &tmC, &tmH, &tmY, dt, A, Dv, L, H, G, T, hgs, ksplit, b, c,
                         t, hg * hgs, smem, progress, HP, false, status);
    }
}

template <int Q, int N, int HP>
cudaError_t launch_impl(const void* x, const float* dt, const float* A, const void* B,
                        const void* C, const float* D, const float* init, void* prev, void* y,
                        float* fin, int* sched, const Dims& d, int ksplit, int pc,
                        const Cfg& cf, cudaStream_t s) {
    using FS = FusedSmem<Q, N, HP>;
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

    const int64_t nwalk = walkers(d, HP);
    const int64_t grid = nwalk + out_tiles(d, cf);
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    e = cudaMemsetAsync(sched, 0, (size_t)(32 + nwalk) * sizeof(int), s);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(walk_out_tc_kernel<Q, N, HP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, FS::kAlloc);
    if (e != cudaSuccess) return e;
    walk_out_tc_kernel<Q, N, HP><<<(unsigned)grid, kThreads, FS::kAlloc, s>>>(
        tmXw, tmBw, tmX, tmB, tmC, tmH, tmY, dt, A, D, init, static_cast<__nv_bfloat16*>(prev), fin,
        d.L, (int)d.H, (int)d.G, d.T, cf.hg, cf.hg2, cf.ks, ksplit, pc, sched, (int)nwalk, status);
    return cudaGetLastError();
}

}  // namespace

bool walk_out_supported(const Dims& d) {
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    return (v.N == 128 || v.N == 64) && (v.Q == 128 || v.Q == 256) &&
           walkers(v, 2) <= 0x7fffffffLL;
}

bool walk_out_preferred(const Dims& d) {
    // The overlap pays once the walk is long enough: the output tiles of the
    // last chunk start only when the walk ends (measured: 8 chunks even to 2 %
    // ahead, 16 and 32 chunks 10-14 % ahead, 4 chunks behind); with more
    // walkers than SMs the walk runs in waves and tiles start only after the
    // last wave.
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    return walk_out_supported(d) && d.T >= 8 && walkers(v, config(v).hp) <= 160;
}

size_t walk_out_sched_bytes(const Dims& d) {
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    return (size_t)(32 + walkers(v, config(v).hp)) * sizeof(int);
}

cudaError_t launch_walk_out_tc(const void* x, const float* dt, const float* A, const void* B,
                               const void* C, const float* D, const float* init, void* prev,
                               void* y, float* final_states, int* sched, const Dims& d,
                               cudaStream_t s) {
    if (!walk_out_supported(d)) return cudaErrorNotSupported;
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    const Cfg cf = config(v);
    const int pc = head_cols(d);
#define SSD_WALK_OUT(Q_, N_, HP_)                                                             \
    if (v.Q == Q_ && v.N == N_ && cf.hp == HP_)                                               \
        return launch_impl<Q_, N_, HP_>(x, dt, A, B, C, D, init, prev, y, final_states, sched, v, \
                                        k, pc, cf, s);
    SSD_WALK_OUT(256, 128, 4)
    SSD_WALK_OUT(128, 128, 4)
    SSD_WALK_OUT(256, 64, 2)
    SSD_WALK_OUT(128, 64, 2)
#undef SSD_WALK_OUT
    return cudaErrorNotSupported;
}

}  // namespace ssd
