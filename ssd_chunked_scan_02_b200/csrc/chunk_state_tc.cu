// chunk_state_tc.cu -- chunk states on the tcgen05 tensor cores (bf16 inputs,
// fp32 accumulation), steps a0 + a2 of the block-decomposed SSD forward:
//
//   cs_j  = sum_{k <= j} dt_k A_h           (inclusive prefix, fp32, warp shuffles)
//   w_j   = exp(cs_last - cs_j) dt_j        (decay to the chunk's end, times dt)
//   S[p, n] = sum_j (w_j x_j[p]) B_j[n]    (P x N chunk state, zero start)
//
// "Transformers are SSMs" (CiteArk), AI research summary: the state a chunk
// hands on is one dense contraction over the chunk's tokens (B^T (w * X)),
// which is what the tensor cores are for.
//
// One CTA per (batch, chunk, HP consecutive head pairs of one B/C group).
// Per head pair one MMA group over K = chunk tokens.  With dstate N = 128 it
// computes S^T (M = N state rows, N = two heads x P = 64 columns): A = the
// chunk's B tile, B = the two heads' scaled x tiles, so a TMEM lane is a
// state column n and the epilogue's stores of S[p][n] are contiguous across
// a warp.  With N = 64 it computes S (M = two heads x P rows, N = dstate).
// Both operands are MN-major 128-byte-swizzled tiles brought by TMA; the B
// tile is loaded once per CTA.  The work is pipelined over head pairs by
// warp role:
//   warp 12 (one lane)  TMA producer: B once, then x tiles of the pairs into
//                       a two-slot ring;
//   warps 0-7           dt staging and prefix sums for all heads up front,
//                       then per pair: scale the x rows in place by w_j (the
//                       MMA sees bf16(w_j x_j));
//   warp 13 (one lane)  MMA issuer (and TMEM owner), two accumulator slots;
//   warps 8-11          epilogue: TMEM -> fp32 S in HBM, layout (b, T, H, P, N).
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

constexpr int kThreads = 448;
constexpr int kMaxPairs = 4;

template <int Q, int N>
struct StateSmem {
    static constexpr int kXTile = Q * 128;                 // one head's x tile (Q rows x 64 bf16)
    static constexpr int kB = 0;                           // N/64 blocks of Q rows x 128 B
    static constexpr int kBBytes = (N / 64) * Q * 128;
    static constexpr int kX = kB + kBBytes;                // [2 slots][2 heads] x tiles
    static constexpr int kDt = kX + 4 * kXTile;            // float [2 kMaxPairs][Q]: dt
    static constexpr int kW = kDt + 2 * kMaxPairs * Q * 4; // float [2 kMaxPairs][Q]: w_j
    static constexpr int kA = kW + 2 * kMaxPairs * Q * 4;  // float [2 kMaxPairs]: A_h
    static constexpr int kBar = kA + 2 * kMaxPairs * 4;
    static constexpr int kTmem = kBar + 16 * 8;
    static constexpr int kFlags = kTmem + 16;
    static constexpr int kTotal = kFlags + 16;
    static constexpr int kAlloc = kTotal + 1024;           // slack to align the base to 1 KB
    static constexpr uint32_t kTmemCols = (2 * N <= 128) ? 128 : 256;   // two fp32 D slots
};

enum {
    BAR_B = 0, BAR_XFULL = 1, BAR_XSCALED = 3, BAR_XEMPTY = 5, BAR_ACCFULL = 7, BAR_ACCEMPTY = 9,
    BAR_COUNT = 11
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int Q, int N>
__global__ void __launch_bounds__(kThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmB, const float* __restrict__ dt,
                      const float* __restrict__ A, float* __restrict__ states,
                      float* __restrict__ logdecay, int64_t L, int H, int G, int64_t T, int HP,
                      WaitCtx status) {
    using S = StateSmem<Q, N>;
    constexpr bool kTrans = (N == 128);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sB = smem + S::kB;
    uint8_t* sX = smem + S::kX;
    float* s_dt = reinterpret_cast<float*>(smem + S::kDt);
    float* s_w = reinterpret_cast<float*>(smem + S::kW);
    float* s_A = reinterpret_cast<float*>(smem + S::kA);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + S::kFlags);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bt = blockIdx.x;
    const int64_t c = bt % T, b = bt / T;
    const int pair0 = blockIdx.y * HP;
    const int g = (2 * pair0) / (H / G);
    const int64_t t0 = c * Q;
    const int len = (int)((L - t0) < Q ? (L - t0) : Q);

    if (tid == 0) {
        for (int i = 0; i < BAR_COUNT; ++i) mbar_init(&bars[i], 1);
        s_flag[0] = 0;
        fence_mbar_init();
    }
    if (warp == 13) {
        tmem_alloc(s_tmem, S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 12) {
        // ================================================== TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmB);
            mbar_expect_tx(&bars[BAR_B], S::kBBytes);
            for (int nb = 0; nb < N / 64; ++nb)
                tma_load_4d(sB + nb * Q * 128, &tmB, &bars[BAR_B], nb * 64, g, (int)t0, (int)b);
            bool ok = true;
            for (int pi = 0; pi < HP && ok; ++pi) {
                const int s = pi & 1;
                if (pi >= 2)
                    ok = mbar_wait(&bars[BAR_XEMPTY + s], (uint32_t)(((pi >> 1) - 1) & 1), status);
                if (!ok) break;
                const int h0 = 2 * (pair0 + pi);
                mbar_expect_tx(&bars[BAR_XFULL + s], 2 * S::kXTile);
                tma_load_4d(sX + (2 * s + 0) * S::kXTile, &tmX, &bars[BAR_XFULL + s], 0, h0,
                            (int)t0, (int)b);
                tma_load_4d(sX + (2 * s + 1) * S::kXTile, &tmX, &bars[BAR_XFULL + s], 0, h0 + 1,
                            (int)t0, (int)b);
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp == 13) {
        // ================================================== MMA issuer
        if (lane == 0) {
            // N = 128: D = S^T = B^T (w x) (M = 128 state rows, N = 128 pair columns);
            // N = 64:  D = S   = (w x)^T B (M = 128 pair rows, N = 64 state columns).
            constexpr uint32_t kIdesc = idesc_bf16_f32(128, kTrans ? 128 : N, true, true);
            bool ok = mbar_wait(&bars[BAR_B], 0, status);
            for (int pi = 0; pi < HP && ok; ++pi) {
                const int s = pi & 1;
                ok = mbar_wait(&bars[BAR_XSCALED + s], (uint32_t)((pi >> 1) & 1), status) &&
                     (pi < 2 || mbar_wait(&bars[BAR_ACCEMPTY + s], (uint32_t)(((pi >> 1) - 1) & 1),
                                          status));
                if (!ok) break;
                tc_fence_after();
                const uint32_t x0 = smem_u32(sX + (2 * s) * S::kXTile);
                const uint32_t b0 = smem_u32(sB);
                for (int ks = 0; ks < Q / 16; ++ks) {
                    // x pair: two 64-column atoms (heads) kXTile apart; B: 64-column
                    // atoms of dstate Q * 128 apart; 8-row groups 1024 B apart.
                    const uint64_t xd = smem_desc_sw128(x0 + ks * 2048, S::kXTile, 1024);
                    const uint64_t bd = smem_desc_sw128(b0 + ks * 2048, Q * 128, 1024);
                    if (kTrans) mma_ss(tmem + s * 128, bd, xd, kIdesc, ks > 0);
                    else mma_ss(tmem + s * N, xd, bd, kIdesc, ks > 0);
                }
                mma_commit(&bars[BAR_XEMPTY + s]);
                mma_commit(&bars[BAR_ACCFULL + s]);
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp < 8) {
        // ================================================== dt / scale warps (0-7)
        // (a0) dt of every head of the CTA for the whole chunk in one coalesced
        // pass (the heads of a token are contiguous), then per head the
        // inclusive prefix sum of dt*A and w_j = exp(cs_last - cs_j) dt_j.
        const int nh = 2 * HP;
        for (int e = tid; e < nh * Q; e += 256) {
            const int j = e / nh, k = e - j * nh;
            s_dt[k * Q + j] = (j < len) ? dt[(b * L + t0 + j) * H + 2 * pair0 + k] : 0.f;
        }
        if (tid < nh) s_A[tid] = A[2 * pair0 + tid];
        named_bar_sync(1, 256);
        for (int k = warp; k < nh; k += 8) {
            const float Ah = s_A[k];
            const float* dk = s_dt + k * Q;
            float* wk = s_w + k * Q;
            float carry = 0.f;
            for (int base = 0; base < Q; base += 32) {
                float v = dk[base + lane] * Ah;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_up_sync(0xffffffffu, v, o);
                    if (lane >= o) v += u;
                }
                v += carry;
                wk[base + lane] = v;                     // cs_j for now
                carry = __shfl_sync(0xffffffffu, v, 31);
            }
            const float last = carry;                    // tokens past the sequence end add 0
            __syncwarp();
            for (int j = lane; j < Q; j += 32) wk[j] = expf(last - wk[j]) * dk[j];
            if (lane == 0) logdecay[(b * T + c) * H + 2 * pair0 + k] = last;
        }
        named_bar_sync(1, 256);
        bool fail = false;
        for (int pi = 0; pi < HP; ++pi) {
            const int s = pi & 1;
            fail = !mbar_wait(&bars[BAR_XFULL + s], (uint32_t)((pi >> 1) & 1), status);
            if (named_bar_or(1, 256, fail)) break;
            // (a2 operand) scale each x row j of both heads by w_j, in place
            for (int r = tid; r < 2 * Q; r += 256) {
                const int k = r / Q, j = r - k * Q;
                const float wj = s_w[(2 * pi + k) * Q + j];
                uint4* row = reinterpret_cast<uint4*>(sX + (2 * s + k) * S::kXTile + j * 128);
                uint4 v[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] = row[q];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t* u = reinterpret_cast<uint32_t*>(&v[q]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u[e]));
                        u[e] = pack_bf16x2(f.x * wj, f.y * wj);
                    }
                    row[q] = v[q];
                }
            }
            fence_proxy_async_smem();           // generic writes -> visible to the MMA (async proxy)
            named_bar_sync(1, 256);
            if (tid == 0) mbar_arrive(&bars[BAR_XSCALED + s]);
        }
        if (fail) s_flag[0] = 1;
    } else {
        // ================================================== epilogue warps (8-11)
        const int m = tid - 256;                 // TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        bool fail = false;
        for (int pi = 0; pi < HP; ++pi) {
            const int s = pi & 1;
            fail = !mbar_wait(&bars[BAR_ACCFULL + s], (uint32_t)((pi >> 1) & 1), status);
            if (named_bar_or(2, 128, fail)) break;
            tc_fence_after();
            if (kTrans) {
                // lane m = state column n; column c = (head c / 64, p = c % 64)
                const int n = m;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + s * 128 + cc * 32, r);
                    const int h = 2 * (pair0 + pi) + (cc >> 1);
                    float* out = states + (((b * T + c) * H + h) * 64 + (cc & 1) * 32) * (int64_t)N + n;
#pragma unroll
                    for (int e = 0; e < 32; ++e) out[(int64_t)e * N] = __uint_as_float(r[e]);
                }
            } else {
                // lane m = (head m / 64, p = m % 64); columns = state n
                const int h = 2 * (pair0 + pi) + (m >> 6);
                float* out = states + (((b * T + c) * H + h) * 64 + (m & 63)) * (int64_t)N;
#pragma unroll
                for (int cc = 0; cc < N / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + s * N + cc * 32, r);
                    float4* o4 = reinterpret_cast<float4*>(out + cc * 32);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        o4[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                            __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
                }
            }
            tc_fence_before();
            named_bar_sync(2, 128);
            if (m == 0) mbar_arrive(&bars[BAR_ACCEMPTY + s]);
        }
        if (fail) s_flag[0] = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (s_flag[0] && tid == 12 * 32) {
        // A wait gave up somewhere: give outstanding TMA loads and MMAs a last
        // (bounded) chance to land before the shared memory and TMEM go away.
        mbar_wait(&bars[BAR_B], 0, status);
        for (int k = 0; k < 2; ++k) {
            mbar_wait(&bars[BAR_XFULL + k], 0, status);
            mbar_wait(&bars[BAR_ACCFULL + k], 0, status);
        }
    }
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, S::kTmemCols);
    }
}

int pick_pairs_per_cta(int64_t H, int64_t G) {
    const int64_t pairs_in_group = (H / G) / 2;
    for (int hp = kMaxPairs; hp > 1; --hp)
        if (pairs_in_group % hp == 0) return hp;
    return 1;
}

template <int Q, int N>
cudaError_t launch_impl(const void* x, const float* dt, const float* A, const void* B,
                        float* states, float* logdecay, const Dims& d, cudaStream_t s) {
    using S = StateSmem<Q, N>;
    CUtensorMap tmX, tmB;
    const uint64_t xdims[4] = {64, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t xstr[3] = {64 * 2, (uint64_t)(d.H * 64 * 2), (uint64_t)(d.L * d.H * 64 * 2)};
    const uint32_t xbox[4] = {64, 1, Q, 1};
    cudaError_t e = make_tmap_bf16(&tmX, x, 4, xdims, xstr, xbox);
    if (e != cudaSuccess) return e;
    const uint64_t bdims[4] = {(uint64_t)N, (uint64_t)d.G, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t bstr[3] = {(uint64_t)N * 2, (uint64_t)(d.G * N * 2), (uint64_t)(d.L * d.G * N * 2)};
    const uint32_t bbox[4] = {64, 1, Q, 1};
    e = make_tmap_bf16(&tmB, B, 4, bdims, bstr, bbox);
    if (e != cudaSuccess) return e;
    const sm100::WaitCtx status = make_wait_ctx();
    if (!status.word) return cudaErrorUnknown;

    const int HP = pick_pairs_per_cta(d.H, d.G);
    e = cudaFuncSetAttribute(chunk_state_tc_kernel<Q, N>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(d.b * d.T), (unsigned)(d.H / (2 * HP)));
    chunk_state_tc_kernel<Q, N><<<grid, kThreads, S::kAlloc, s>>>(
        tmX, tmB, dt, A, states, logdecay, d.L, (int)d.H, (int)d.G, d.T, HP, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_state_tc(const void* x, const float* dt, const float* A, const void* B,
                                  float* states, float* logdecay, const Dims& d, cudaStream_t s) {
    if (d.Q == 256 && d.N == 128) return launch_impl<256, 128>(x, dt, A, B, states, logdecay, d, s);
    if (d.Q == 256 && d.N == 64) return launch_impl<256, 64>(x, dt, A, B, states, logdecay, d, s);
    if (d.Q == 128 && d.N == 128) return launch_impl<128, 128>(x, dt, A, B, states, logdecay, d, s);
    if (d.Q == 128 && d.N == 64) return launch_impl<128, 64>(x, dt, A, B, states, logdecay, d, s);
    return cudaErrorNotSupported;
}

}  // namespace ssd
