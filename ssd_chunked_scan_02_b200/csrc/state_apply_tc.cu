// state_apply_tc.cu -- the correction of the sequence-parallel forward on the
// tcgen05 tensor cores (bf16, headdim 64, dstate 64 or 128):
//
//   y_t += alpha_t (h_in C_t),   alpha_t = exp(cs_t) = 2^(prefix_k + cs_t within the tile)
//
// for every token t of a shard and head h, where h_in is the state entering
// the shard.  "Transformers are SSMs" (CiteArk), what this means: the state is
// what carries a sequence forward, so a shard computed from a zero state is
// completed by adding its entering state's contribution -- the same
// contraction as the entering-state term of the forward's chunk outputs,
// C (h_in)^T, taken over the whole shard.
//
// CTA per (batch, 128-token tile, block of HG heads of one group).  Roles
// (192 threads): warp 0 TMA producer (the tile's C rows once, then each
// head's h_in in bf16 through a two-slot ring); warp 1 MMA issuer and TMEM
// owner (ZW = C h^T, M = 128 tokens, N = 64, K = dstate, two accumulators);
// warps 2-5 epilogue (lane = token: the head's decay prefix by warp scans,
// then y row += alpha ZW, rounded once to bf16).  A head whose decay at the
// tile start has underflowed (A <= 0) is skipped by every role alike: its
// correction is exactly zero.  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "seqpar.h"
#include "sm100.cuh"
#include "tc_host.h"
#include "tc_kernels.h"

namespace ssd {
namespace {
using namespace sm100;

constexpr int kThreads = 192;
constexpr int kMaxHeads = 16;
constexpr float kLog2e = 1.4426950408889634f;

template <int N>
struct ApplySmem {
    static constexpr int kNB = N / 64;
    static constexpr int kC = 0;                            // kNB x 128 rows x 128 B
    static constexpr int kH = kC + kNB * 128 * 128;         // 2 slots x kNB x 64 rows x 128 B
    static constexpr int kHTile = kNB * 64 * 128;
    static constexpr int kWs = kH + 2 * kHTile;             // float [2][4]: warp sums of the scan
    static constexpr int kBar = kWs + 32;
    static constexpr int kTmem = kBar + 16 * 8;
    static constexpr int kFlags = kTmem + 16;
    static constexpr int kTotal = kFlags + 16;
    // at least 58 KB, so that no more than four CTAs (4 x 128 TMEM columns)
    // share an SM
    static constexpr int kAlloc = (kTotal + 1024 > 58 * 1024) ? kTotal + 1024 : 58 * 1024;
};

enum { BAR_C = 0, BAR_HFULL = 1, BAR_HEMPTY = 3, BAR_ACCFULL = 5, BAR_ACCEMPTY = 7, BAR_COUNT = 9 };
constexpr uint32_t kTmemCols = 128;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int N>
__global__ void __launch_bounds__(kThreads)
state_apply_tc_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmH,
                      const float* __restrict__ dt, const float* __restrict__ A,
                      const float* __restrict__ tile_prefix, __nv_bfloat16* __restrict__ y,
                      int64_t L, int H, int G, int64_t ntiles, int HG, int ksplit,
                      WaitCtx status) {
    using S = ApplySmem<N>;
    // H counts virtual heads (headdim 64); real head = virtual head / ksplit
    const int Hr = H / ksplit;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bk = blockIdx.x;
    const int64_t k = bk % ntiles, b = bk / ntiles;
    const int head0 = blockIdx.y * HG;
    const int g = head0 / (H / G);
    const int64_t t0 = k * 128;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sC = smem + S::kC;
    uint8_t* sH = smem + S::kH;
    float* s_ws = reinterpret_cast<float*>(smem + S::kWs);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + S::kFlags);

    // which heads of the block have a non-zero correction on this tile (every
    // role reads the same values, so all agree)
    uint32_t active = 0;
    for (int hi = 0; hi < HG; ++hi) {
        const float a = A[(head0 + hi) / ksplit];
        const float pre = tile_prefix[(b * ntiles + k) * Hr + (head0 + hi) / ksplit];
        if (!(a <= 0.f && exp2f(pre) == 0.f)) active |= 1u << hi;
    }
    if (active == 0) return;

    if (tid == 0) {
        for (int i = 0; i < BAR_COUNT; ++i) mbar_init(&bars[i], 1);
        s_flag[0] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ================================================== TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmC);
            prefetch_tmap(&tmH);
            mbar_expect_tx(&bars[BAR_C], (uint32_t)(S::kNB * 128 * 128));
            for (int nb = 0; nb < S::kNB; ++nb)
                tma_load_4d(sC + nb * 128 * 128, &tmC, &bars[BAR_C], nb * 64, g, (int)t0, (int)b);
            bool ok = true;
            int j = 0;
            for (int hi = 0; hi < HG && ok; ++hi) {
                if (!(active >> hi & 1)) continue;
                const int s = j & 1;
                if (j >= 2) ok = mbar_wait(&bars[BAR_HEMPTY + s], (uint32_t)(((j >> 1) - 1) & 1), status);
                if (!ok) break;
                mbar_expect_tx(&bars[BAR_HFULL + s], (uint32_t)S::kHTile);
                const int hrow = (int)((b * H + head0 + hi) * 64);
                for (int nb = 0; nb < S::kNB; ++nb)
                    tma_load_2d(sH + s * S::kHTile + nb * 64 * 128, &tmH, &bars[BAR_HFULL + s],
                                nb * 64, hrow);
                ++j;
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp == 1) {
        // ================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdesc = idesc_bf16_f32(128, 64, false, false);   // C, h K-major
            bool ok = mbar_wait(&bars[BAR_C], 0, status);
            const uint64_t cd = smem_desc_sw128(smem_u32(sC), 16, 1024);
            int j = 0;
            for (int hi = 0; hi < HG && ok; ++hi) {
                if (!(active >> hi & 1)) continue;
                const int s = j & 1;
                ok = mbar_wait(&bars[BAR_HFULL + s], (uint32_t)((j >> 1) & 1), status) &&
                     (j < 2 || mbar_wait(&bars[BAR_ACCEMPTY + s], (uint32_t)(((j >> 1) - 1) & 1), status));
                if (!ok) break;
                tc_fence_after();
                const uint64_t hd = smem_desc_sw128(smem_u32(sH + s * S::kHTile), 16, 1024);
                const uint32_t acc = tmem + 64 * s;
#pragma unroll
                for (int ks = 0; ks < N / 16; ++ks)
                    mma_ss(acc, cd + (uint64_t)((ks >> 2) * 1024 + (ks & 3) * 2),
                           hd + (uint64_t)((ks >> 2) * 512 + (ks & 3) * 2), kIdesc, ks > 0);
                mma_commit(&bars[BAR_HEMPTY + s]);
                mma_commit(&bars[BAR_ACCFULL + s]);
                ++j;
            }
            if (!ok) s_flag[0] = 1;
        }
    } else {
        // ================================================== epilogue (warps 2-5)
        // Per head: the decay prefix from dt (loaded a head ahead), the y row
        // loaded before the accumulator is waited for, then y += alpha ZW.
        const int q = warp & 3;                    // TMEM lane quarter (warps 2,3,4,5 -> 2,3,0,1)
        const int m = q * 32 + lane;               // token row of the tile
        const int64_t t = t0 + m;
        const bool in = t < L;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float* dt_row = dt + (b * L + (in ? t : 0)) * Hr;
        bool fail = false;
        int j = 0;
        int hi = __ffs(active) - 1;                // first active head
        float dtv = in ? dt_row[(head0 + hi) / ksplit] : 0.f;
        for (; hi < HG; ++j) {
            const int s = j & 1;
            const int h = head0 + hi;
            const int hn = (hi + 1 < HG && (active >> (hi + 1))) ? hi + __ffs(active >> (hi + 1)) : HG;
            // this head's y row, in flight while the scan and the MMA finish
            uint4 yv[8];
            uint4* yr = reinterpret_cast<uint4*>(y + ((b * L + t) * H + h) * 64);
            if (in) {
#pragma unroll
                for (int c = 0; c < 8; ++c) yv[c] = yr[c];
            }
            // alpha_m = 2^(prefix + inclusive sum over the tile's tokens <= m)
            float v = dtv * (A[h / ksplit] * kLog2e);
            if (hn < HG) dtv = in ? dt_row[(head0 + hn) / ksplit] : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (lane == 31) s_ws[s * 4 + q] = v;
            fail = !mbar_wait(&bars[BAR_ACCFULL + s], (uint32_t)((j >> 1) & 1), status);
            if (named_bar_or(1, 128, fail)) {
                fail = true;
                break;
            }
            tc_fence_after();
            float off = tile_prefix[(b * ntiles + k) * Hr + h / ksplit];
            for (int w = 0; w < q; ++w) off += s_ws[s * 4 + w];
            const float al = exp2f(off + v);
            uint32_t zr[32], zr2[32];
            tmem_ld32x2(tmem + lane_base + 64 * s, tmem + lane_base + 64 * s + 32, zr, zr2);
            // the accumulator has been read: the MMA may reuse it
            tc_fence_before();
            named_bar_sync(1, 128);
            if (m == 0) mbar_arrive(&bars[BAR_ACCEMPTY + s]);
            if (in) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t* w = reinterpret_cast<uint32_t*>(&yv[c]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = 8 * c + 2 * e;
                        const float z0 = __uint_as_float(col < 32 ? zr[col] : zr2[col - 32]);
                        const float z1 = __uint_as_float(col + 1 < 32 ? zr[col + 1] : zr2[col - 31]);
                        const float2 yf = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
                        w[e] = pack_bf16x2(fmaf(al, z0, yf.x), fmaf(al, z1, yf.y));
                    }
                    yr[c] = yv[c];
                }
            }
            hi = hn;
        }
        if (fail) s_flag[0] = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (s_flag[0] && tid == 0) {
        // A wait gave up somewhere: give outstanding TMA loads and MMAs a last
        // (bounded) chance to land before the shared memory and TMEM go away.
        mbar_wait(&bars[BAR_C], 0, status);
        for (int s = 0; s < 2; ++s) mbar_wait(&bars[BAR_HFULL + s], 0, status);
        for (int s = 0; s < 2; ++s) mbar_wait(&bars[BAR_ACCFULL + s], 0, status);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

int pick_heads(int64_t H, int64_t G) {
    const int64_t hpg = H / G;
    for (int hg = kMaxHeads; hg > 1; --hg)
        if (hpg % hg == 0) return hg;
    return 1;
}

template <int N>
cudaError_t launch_impl(const __nv_bfloat16* h_bf16, const float* dt, const float* A,
                        const void* C, const float* tile_prefix, void* y, const Dims& d,
                        int ksplit, cudaStream_t s) {
    using S = ApplySmem<N>;
    CUtensorMap tmC, tmH;
    const uint64_t cdims[4] = {(uint64_t)N, (uint64_t)d.G, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t cstr[3] = {(uint64_t)N * 2, (uint64_t)(d.G * N * 2), (uint64_t)(d.L * d.G * N * 2)};
    const uint32_t cbox[4] = {64, 1, 128, 1};
    cudaError_t e = make_tmap_bf16(&tmC, C, 4, cdims, cstr, cbox);
    if (e != cudaSuccess) return e;
    const uint64_t hdims[2] = {(uint64_t)N, (uint64_t)(d.b * d.H * 64)};
    const uint64_t hstr[1] = {(uint64_t)N * 2};
    const uint32_t hbox[2] = {64, 64};
    e = make_tmap_bf16(&tmH, h_bf16, 2, hdims, hstr, hbox);
    if (e != cudaSuccess) return e;
    const sm100::WaitCtx status = make_wait_ctx();
    if (!status.word) return cudaErrorUnknown;
    const int HG = pick_heads(d.H, d.G);
    e = cudaFuncSetAttribute(state_apply_tc_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             S::kAlloc);
    if (e != cudaSuccess) return e;
    const int64_t nt = correction_tiles(d);
    dim3 grid((unsigned)(d.b * nt), (unsigned)(d.H / HG));
    state_apply_tc_kernel<N><<<grid, kThreads, S::kAlloc, s>>>(
        tmC, tmH, dt, A, tile_prefix, static_cast<__nv_bfloat16*>(y), d.L, (int)d.H, (int)d.G, nt,
        HG, ksplit, status);
    return cudaGetLastError();
}

}  // namespace

bool correction_tc_supported(const Dims& d, Elt t) {
    return t == Elt::BF16 && d.P % 64 == 0 && d.P <= 256 && (d.N == 64 || d.N == 128) &&
           d.b > 0 && d.L > 0 && d.L <= 0x7fffffffLL && d.b * d.H * d.P <= 0x7fffffffLL;
}

cudaError_t launch_correction_tc(const __nv_bfloat16* h_bf16, const float* dt, const float* A,
                                 const void* C, const float* tile_prefix, void* y, const Dims& d,
                                 cudaStream_t s) {
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    if (v.N == 128) return launch_impl<128>(h_bf16, dt, A, C, tile_prefix, y, v, k, s);
    if (v.N == 64) return launch_impl<64>(h_bf16, dt, A, C, tile_prefix, y, v, k, s);
    return cudaErrorNotSupported;
}

}  // namespace ssd
