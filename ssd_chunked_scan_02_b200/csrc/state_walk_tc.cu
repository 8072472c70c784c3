// state_walk_tc.cu -- chunk states and the inter-chunk recurrence in one pass
// (steps a0 + a2 + a3 of the block-decomposed SSD forward, bf16 inputs):
//
//   h_{-1} = init (or 0);  for each chunk c:  prev_c = h_{c-1}   (written, bf16)
//                                            h_c = exp(cs_last) h_{c-1} + S_c
//   S_c = sum_j (exp(cs_last - cs_j) dt_j x_j) B_j^T   (tensor cores, fp32 accumulation)
//
// "论文解读：Mamba: ...", 状态空间模型: the linear-recurrence form, taken one
// chunk per step; "Transformers are SSMs" (CiteArk), AI research summary: the
// chunk's contribution is one dense contraction.
//
// One CTA per (batch, head pair) walks the chunks in order.  The running
// state lives in TMEM (fp32, 128 columns): before chunk c's MMAs the
// epilogue warps read h_{c-1}, write it out as the chunk's entering state,
// scale it by the chunk decay and store it back; the MMAs of chunk c then
// accumulate S_c on top of it.  Nothing else of the state ever leaves the
// chip (no per-chunk fp32 states in HBM).  With dstate N = 128 the MMA forms
// h^T (M = 128 state rows, N = two heads x P = 64), so a TMEM lane is a state
// column and the state writes are contiguous across a warp; with N = 64 it
// forms h (M = two heads x P rows, N = 64).  x and B come by TMA in 64-token
// sub-steps through a three-entry ring (x scaled in place by the decay
// weights before the MMA reads it).  Sized for two CTAs per SM (~105 KB of
// shared memory, 128 TMEM columns each).
//
// Roles (320 threads): warps 0-3 dt prefix sums and x scaling; warps 4-7
// state epilogue; warp 8 TMA producer; warp 9 MMA issuer and TMEM owner.
// Every wait is bounded; a warpgroup leaves its loop only when all its
// threads agree (bar.red.or).
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"
#include "ssd_internal.h"
#include "tc_host.h"
#include "tc_kernels.h"

namespace ssd {
namespace {
using namespace sm100;

constexpr int kThreads = 320;
constexpr int kStages = 3;
constexpr int kSub = 64;                 // tokens per ring entry

template <int Q, int N>
struct WalkSmem {
    static constexpr int kXPart = 2 * kSub * 128;          // two heads x 64 rows x 128 B
    static constexpr int kBPart = (N / 64) * kSub * 128;   // N/64 blocks x 64 rows x 128 B
    static constexpr int kEntry = kXPart + kBPart;
    static constexpr int kRing = 0;
    static constexpr int kDt = kRing + kStages * kEntry;   // float [2 buf][2 heads][Q]
    static constexpr int kW = kDt + 2 * 2 * Q * 4;         // float [2 buf][2 heads][Q]
    static constexpr int kA = kW + 2 * 2 * Q * 4;          // float [2 buf][2]: chunk decays
    static constexpr int kBar = kA + 64;
    static constexpr int kTmem = kBar + 16 * 8;
    static constexpr int kFlags = kTmem + 16;
    static constexpr int kTotal = kFlags + 16;
    static constexpr int kAlloc = kTotal + 1024;
};

enum {
    BAR_FULL = 0, BAR_EMPTY = 3, BAR_SCALED = 6, BAR_AREADY = 9, BAR_AFREE = 11, BAR_HREADY = 13,
    BAR_MMADONE = 14, BAR_COUNT = 15
};
constexpr uint32_t kTmemCols = 128;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int Q, int N>
__global__ void __launch_bounds__(kThreads, 2)
state_walk_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                     const float* __restrict__ dt, const float* __restrict__ A,
                     const float* __restrict__ init, __nv_bfloat16* __restrict__ prev,
                     float* __restrict__ fin, int64_t L, int H, int G, int64_t T,
                     WaitCtx status) {
    using S = WalkSmem<Q, N>;
    constexpr bool kTrans = (N == 128);
    constexpr int kNSub = Q / kSub;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t b = blockIdx.x / (H / 2);
    const int h0 = 2 * (int)(blockIdx.x % (H / 2));
    const int g = h0 / (H / G);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* ring = smem + S::kRing;
    float* s_dt = reinterpret_cast<float*>(smem + S::kDt);
    float* s_w = reinterpret_cast<float*>(smem + S::kW);
    float* s_a = reinterpret_cast<float*>(smem + S::kA);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + S::kFlags);

    if (tid == 0) {
        for (int i = 0; i < BAR_COUNT; ++i) mbar_init(&bars[i], 1);
        s_flag[0] = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int64_t nsteps = T * kNSub;

    if (warp == 8) {
        // ================================================== TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmB);
            bool ok = true;
            for (int64_t si = 0; si < nsteps && ok; ++si) {
                const int e = (int)(si % kStages);
                const int64_t u = si / kStages;
                if (u >= 1) ok = mbar_wait(&bars[BAR_EMPTY + e], (uint32_t)((u - 1) & 1), status);
                if (!ok) break;
                const int row = (int)((si / kNSub) * Q + (si % kNSub) * kSub);
                uint8_t* ent = ring + e * S::kEntry;
                mbar_expect_tx(&bars[BAR_FULL + e], S::kEntry);
                tma_load_4d(ent, &tmX, &bars[BAR_FULL + e], 0, h0, row, (int)b);
                tma_load_4d(ent + kSub * 128, &tmX, &bars[BAR_FULL + e], 0, h0 + 1, row, (int)b);
                for (int nb = 0; nb < N / 64; ++nb)
                    tma_load_4d(ent + S::kXPart + nb * kSub * 128, &tmB, &bars[BAR_FULL + e],
                                nb * 64, g, row, (int)b);
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp == 9) {
        // ================================================== MMA issuer
        if (lane == 0) {
            // N = 128: h^T (M = 128 state rows, N = 128 pair columns) += B^T (w x)
            // N = 64:  h   (M = 128 pair rows,  N = 64 state columns) += (w x)^T B
            constexpr uint32_t kIdesc = idesc_bf16_f32(128, kTrans ? 128 : N, true, true);
            bool ok = true;
            int64_t si = 0;
            for (int64_t c = 0; c < T && ok; ++c) {
                ok = mbar_wait(&bars[BAR_HREADY], (uint32_t)(c & 1), status);
                for (int sub = 0; sub < kNSub && ok; ++sub, ++si) {
                    const int e = (int)(si % kStages);
                    const int64_t u = si / kStages;
                    ok = mbar_wait(&bars[BAR_SCALED + e], (uint32_t)(u & 1), status);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t x0 = smem_u32(ring + e * S::kEntry);
                    const uint32_t b0 = x0 + S::kXPart;
                    for (int ks = 0; ks < kSub / 16; ++ks) {
                        // x pair: two 64-column atoms (heads) 8 KB apart; B: 64-column
                        // atoms of dstate 8 KB apart; 8-row groups 1024 B apart.
                        const uint64_t xd = smem_desc_sw128(x0 + ks * 2048, kSub * 128, 1024);
                        const uint64_t bd = smem_desc_sw128(b0 + ks * 2048, kSub * 128, 1024);
                        if (kTrans) mma_ss(tmem, bd, xd, kIdesc, true);
                        else mma_ss(tmem, xd, bd, kIdesc, true);
                    }
                    mma_commit(&bars[BAR_EMPTY + e]);
                }
                if (ok) mma_commit(&bars[BAR_MMADONE]);
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp < 4) {
        // ================================================== dt prefix sums and x scaling
        // Each thread prefetches 2 Q / 128 dt values of the next chunk into
        // registers while the current chunk is processed.
        constexpr int kPer = 2 * Q / 128;
        float pre[kPer];
        auto load_dt = [&](int64_t c) {
#pragma unroll
            for (int r = 0; r < kPer; ++r) {
                const int e = tid + 128 * r;
                const int j = e >> 1, k = e & 1;
                const int64_t tok = c * Q + j;
                pre[r] = (tok < L) ? dt[(b * L + tok) * H + h0 + k] : 0.f;
            }
        };
        load_dt(0);
        const float Ak = (warp < 2) ? A[h0 + warp] : 0.f;
        bool fail = false;
        int64_t si = 0;
        for (int64_t c = 0; c < T; ++c) {
            const int cb = (int)(c & 1);
            // buffer cb is free once the epilogue has read chunk c-2's decays
            fail = named_bar_or(1, 128, c >= 2 && !mbar_wait(&bars[BAR_AFREE + cb],
                                                             (uint32_t)(((c >> 1) - 1) & 1), status));
            if (fail) break;
            float* dtb = s_dt + cb * 2 * Q;
            float* wb = s_w + cb * 2 * Q;
#pragma unroll
            for (int r = 0; r < kPer; ++r) {
                const int e = tid + 128 * r;
                dtb[(e & 1) * Q + (e >> 1)] = pre[r];
            }
            if (c + 1 < T) load_dt(c + 1);
            named_bar_sync(1, 128);
            if (warp < 2) {
                const float* dk = dtb + warp * Q;
                float* wk = wb + warp * Q;
                float carry = 0.f;
                for (int base = 0; base < Q; base += 32) {
                    float v = dk[base + lane] * Ak;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float uu = __shfl_up_sync(0xffffffffu, v, o);
                        if (lane >= o) v += uu;
                    }
                    v += carry;
                    wk[base + lane] = v;                    // cs_j for now
                    carry = __shfl_sync(0xffffffffu, v, 31);
                }
                const float last = carry;                   // tokens past the end add 0
                __syncwarp();
                for (int j = lane; j < Q; j += 32) wk[j] = expf(last - wk[j]) * dk[j];
                if (lane == 0) s_a[cb * 2 + warp] = expf(last);
            }
            named_bar_sync(1, 128);
            if (tid == 0) mbar_arrive(&bars[BAR_AREADY + cb]);
            for (int sub = 0; sub < kNSub; ++sub, ++si) {
                const int e = (int)(si % kStages);
                const int64_t u = si / kStages;
                fail = named_bar_or(1, 128, !mbar_wait(&bars[BAR_FULL + e], (uint32_t)(u & 1), status));
                if (fail) break;                              // the same answer in every thread
                // row tid of the entry: head tid / 64, token sub * 64 + tid % 64
                {
                    const int k = tid >> 6, jl = tid & 63;
                    const float wj = wb[k * Q + sub * kSub + jl];
                    uint4* row = reinterpret_cast<uint4*>(ring + e * S::kEntry + k * kSub * 128 + jl * 128);
                    uint4 v[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) v[q] = row[q];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint32_t* uw = reinterpret_cast<uint32_t*>(&v[q]);
#pragma unroll
                        for (int ee = 0; ee < 4; ++ee) {
                            const float2 f =
                                __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&uw[ee]));
                            uw[ee] = pack_bf16x2(f.x * wj, f.y * wj);
                        }
                        row[q] = v[q];
                    }
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (tid == 0) mbar_arrive(&bars[BAR_SCALED + e]);
            }
            if (fail) break;
        }
        if (fail) s_flag[0] = 1;
    } else {
        // ================================================== state epilogue (warps 4-7)
        const int m = tid - 128;                       // TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        bool fail = false;
        for (int64_t c = 0; c <= T; ++c) {
            const int cb = (int)(c & 1);
            // h_{c-1}: the initial state, or the MMA result of chunk c-1
            if (c > 0) fail = !mbar_wait(&bars[BAR_MMADONE], (uint32_t)((c - 1) & 1), status);
            if (c < T)
                fail = fail || !mbar_wait(&bars[BAR_AREADY + cb], (uint32_t)((c >> 1) & 1), status);
            if (named_bar_or(2, 128, fail)) break;
            tc_fence_after();
            float a0 = 1.f, a1 = 1.f;
            if (c < T) {
                a0 = s_a[cb * 2 + 0];
                a1 = s_a[cb * 2 + 1];
            }
            named_bar_sync(2, 128);
            if (c < T && m == 0) mbar_arrive(&bars[BAR_AFREE + cb]);
            if (kTrans) {
                // lane m = state column n; TMEM column cc*32+e = (head cc/2, p = (cc&1)*32 + e)
                const int n = m;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    const int k = cc >> 1, p0 = (cc & 1) * 32;
                    const int64_t srow = ((b * H + h0 + k) * 64 + p0) * (int64_t)N + n;
                    uint32_t r[32];
                    if (c == 0) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r[e] = __float_as_uint(init ? init[srow + (int64_t)e * N] : 0.f);
                    } else {
                        tmem_ld32(tmem + lane_base + cc * 32, r);
                    }
                    if (c < T) {
                        __nv_bfloat16* pr = prev + (((b * T + c) * H + h0 + k) * 64 + p0) * (int64_t)N + n;
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            pr[(int64_t)e * N] = __float2bfloat16_rn(__uint_as_float(r[e]));
                        const float a = k ? a1 : a0;
                        uint32_t lo[16], hi[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            lo[e] = __float_as_uint(a * __uint_as_float(r[e]));
                            hi[e] = __float_as_uint(a * __uint_as_float(r[16 + e]));
                        }
                        tmem_st16(tmem + lane_base + cc * 32, lo);
                        tmem_st16(tmem + lane_base + cc * 32 + 16, hi);
                    } else if (fin) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) fin[srow + (int64_t)e * N] = __uint_as_float(r[e]);
                    }
                }
            } else {
                // lane m = (head m / 64, p = m % 64); TMEM columns = state n (N = 64)
                const int k = m >> 6, p = m & 63;
                const int64_t srow = ((b * H + h0 + k) * 64 + p) * (int64_t)N;
#pragma unroll 1
                for (int cc = 0; cc < N / 32; ++cc) {
                    uint32_t r[32];
                    if (c == 0) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r[e] = __float_as_uint(init ? init[srow + cc * 32 + e] : 0.f);
                    } else {
                        tmem_ld32(tmem + lane_base + cc * 32, r);
                    }
                    if (c < T) {
                        __nv_bfloat16* pr = prev + (((b * T + c) * H + h0 + k) * 64 + p) * (int64_t)N + cc * 32;
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));
                            v.y = pack_bf16x2(__uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
                            v.z = pack_bf16x2(__uint_as_float(r[e + 4]), __uint_as_float(r[e + 5]));
                            v.w = pack_bf16x2(__uint_as_float(r[e + 6]), __uint_as_float(r[e + 7]));
                            *reinterpret_cast<uint4*>(pr + e) = v;
                        }
                        const float a = k ? a1 : a0;
                        uint32_t lo[16], hi[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            lo[e] = __float_as_uint(a * __uint_as_float(r[e]));
                            hi[e] = __float_as_uint(a * __uint_as_float(r[16 + e]));
                        }
                        tmem_st16(tmem + lane_base + cc * 32, lo);
                        tmem_st16(tmem + lane_base + cc * 32 + 16, hi);
                    } else if (fin) {
                        float4* f4 = reinterpret_cast<float4*>(fin + srow + cc * 32);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            f4[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                                __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(2, 128);
            if (c < T && m == 0) mbar_arrive(&bars[BAR_HREADY]);
        }
        if (fail) s_flag[0] = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (s_flag[0] && tid == 8 * 32) {
        // A wait gave up somewhere: give outstanding TMA loads and MMAs a last
        // (bounded) chance to land before the shared memory and TMEM go away.
        for (int k = 0; k < kStages; ++k) mbar_wait(&bars[BAR_FULL + k], 0, status);
        mbar_wait(&bars[BAR_MMADONE], 0, status);
    }
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int Q, int N>
cudaError_t launch_impl(const void* x, const float* dt, const float* A, const void* B,
                        const float* init, void* prev, float* fin, const Dims& d, cudaStream_t s) {
    using S = WalkSmem<Q, N>;
    CUtensorMap tmX, tmB;
    const uint64_t xdims[4] = {64, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t xstr[3] = {64 * 2, (uint64_t)(d.H * 64 * 2), (uint64_t)(d.L * d.H * 64 * 2)};
    const uint32_t box[4] = {64, 1, kSub, 1};
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
    const int64_t grid = d.b * (d.H / 2);
    state_walk_tc_kernel<Q, N><<<(unsigned)grid, kThreads, S::kAlloc, s>>>(
        tmX, tmB, dt, A, init, static_cast<__nv_bfloat16*>(prev), fin, d.L, (int)d.H, (int)d.G,
        d.T, status);
    return cudaGetLastError();
}

}  // namespace

bool walk_preferred(const Dims& d) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // one walker per (batch, head pair): worth it when the walkers alone fill the GPU
    return d.b * (d.H / 2) >= sms && d.b * (d.H / 2) <= 0x7fffffffLL;
}

cudaError_t launch_state_walk_tc(const void* x, const float* dt, const float* A, const void* B,
                                 const float* init, void* prev, float* fin, const Dims& d,
                                 cudaStream_t s) {
    if (d.Q == 256 && d.N == 128) return launch_impl<256, 128>(x, dt, A, B, init, prev, fin, d, s);
    if (d.Q == 256 && d.N == 64) return launch_impl<256, 64>(x, dt, A, B, init, prev, fin, d, s);
    if (d.Q == 128 && d.N == 128) return launch_impl<128, 128>(x, dt, A, B, init, prev, fin, d, s);
    if (d.Q == 128 && d.N == 64) return launch_impl<128, 64>(x, dt, A, B, init, prev, fin, d, s);
    return cudaErrorNotSupported;
}

}  // namespace ssd
