// chunk_out_tc.cu -- chunk outputs on the tcgen05 tensor cores (bf16 inputs,
// fp32 accumulation): steps a1 + a4 of the block-decomposed SSD forward,
//
//   y_i = sum_{j <= i} (C_i . B_j) exp(cs_i - cs_j) dt_j x_j      (masked C B^T term)
//       + exp(cs_i) h_prev C_i                                    (entering state)
//       + D_h x_i                                                 (skip)
//
// "Transformers are SSMs" (CiteArk), what this means: the 1-semiseparable SSM
// restricted to a chunk is structured masked attention, C B^T masked by the
// decay; review page, 核心概念 items 3 and 5; 关键洞察 item 1 (block
// decomposition lets the tensor cores do the work).
//
// One CTA per (batch, chunk, 128-row tile of the chunk, group of HG heads
// that share B and C).  Rows i of the tile need columns j < 128 (t + 1).
//   1. G = C_tile B^T (M = 128, N = 128 (t+1), K = dstate) into TMEM once per
//      CTA; it is shared by the CTA's heads (B, C are per group, not per head).
//   2. Per head: the decay mask is built in registers from the prefix sums of
//      dt*A: on the diagonal 128 x 128 block M_ij = G_ij exp(cs_i - cs_j) dt_j
//      (j <= i); on the block left of it (t = 1) the decay factorises through
//      the block boundary r, M_ij = G_ij * exp(cs_i - r) * (exp(r - cs_j) dt_j),
//      both factors <= 1, so no exponentials per element are needed there.
//      M is written to TMEM as packed bf16 and used as the A operand of
//      Y = M X (kind::f16, A from TMEM, B = x tile from shared memory).
//   3. Z = C_tile h_prev^T (A = C tile, B = the head's entering state, bf16).
//   4. Epilogue: y = Y + exp(cs_i) Z + D_h x, rounded to bf16 once.
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

constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

template <int Q, int N>
struct OutSmem {
    static constexpr int kNB = N / 64;                     // 64-wide blocks of dstate
    static constexpr int kC = 0;                           // kNB x 128 rows x 128 B
    static constexpr int kCBytes = kNB * 128 * 128;
    static constexpr int kB = kC + kCBytes;                // kNB x Q rows x 128 B
    static constexpr int kBBytes = kNB * Q * 128;
    static constexpr int kXTile = Q * 128;                 // x rows [0, Q) of one head
    static constexpr int kX = kB + kBBytes;                // 2 buffers
    static constexpr int kHTile = kNB * 64 * 128;          // h_prev of one head (64 x N)
    static constexpr int kH = kX + 2 * kXTile;             // 2 buffers
    static constexpr int kMaxHeads = 8;                    // heads per CTA (at most)
    static constexpr int kCs = kH + 2 * kHTile;            // float [kMaxHeads][Q] prefix sums (log2 units)
    static constexpr int kDt = kCs + kMaxHeads * Q * 4;    // float [kMaxHeads][Q]
    static constexpr int kBeta = kDt + kMaxHeads * Q * 4;  // float [128]
    static constexpr int kBar = kBeta + 128 * 4;           // 5 mbarriers
    static constexpr int kTmem = kBar + 8 * 8;
    static constexpr int kAbort = kTmem + 4;
    static constexpr int kTotal = kAbort + 4;
    static constexpr int kAlloc = kTotal + 1024;
};

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0;       // fp32 G, up to 256 columns
constexpr uint32_t kColM = 256;     // bf16 mask (A operand), up to 128 columns
constexpr uint32_t kColY = 384;     // fp32 Y, 64 columns
constexpr uint32_t kColZ = 448;     // fp32 Z, 64 columns

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int Q, int N>
__global__ void __launch_bounds__(kThreads, 1)
chunk_out_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmH,
                    const float* __restrict__ dt, const float* __restrict__ A,
                    const float* __restrict__ Dv, __nv_bfloat16* __restrict__ y, int64_t L, int H,
                    int G, int64_t T, int HG, unsigned int* status) {
    using S = OutSmem<Q, N>;
    constexpr int kTiles = Q / 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bx = blockIdx.x;
    const int t = (int)(bx % kTiles);
    const int64_t bt = bx / kTiles;
    const int64_t c = bt % T, b = bt / T;
    const int64_t t0 = c * Q;
    const int len = (int)((L - t0) < Q ? (L - t0) : Q);
    if (128 * t >= len) return;                 // tile entirely past the sequence end
    const int head0 = blockIdx.y * HG;
    const int g = head0 / (H / G);
    const int KJ = 128 * (t + 1);               // columns j this tile needs
    const int row0 = 128 * t;                   // first row of the tile within the chunk

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sC = smem + S::kC;
    uint8_t* sB = smem + S::kB;
    uint8_t* sX = smem + S::kX;
    uint8_t* sH = smem + S::kH;
    float* s_cs = reinterpret_cast<float*>(smem + S::kCs);
    float* s_dt = reinterpret_cast<float*>(smem + S::kDt);
    float* s_beta = reinterpret_cast<float*>(smem + S::kBeta);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);  // 0 BC, 1-2 xh, 3 G, 4 YZ
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + S::kAbort);

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        *s_abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmC);
        prefetch_tmap(&tmH);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

    bool bc_pending = false;
    int g_pending = -1, yz_pending = -1;
    int xh_pending[2] = {-1, -1};
    int xh_issues[2] = {0, 0};

    auto issue_xh = [&](int hi) {
        const int buf = hi & 1;
        const int h = head0 + hi;
        mbar_expect_tx(&bars[1 + buf], (uint32_t)(KJ * 128 + S::kHTile));
        for (int rb = 0; rb <= t; ++rb)
            tma_load_4d(sX + buf * S::kXTile + rb * 128 * 128, &tmX, &bars[1 + buf], 0, h,
                        (int)(t0 + rb * 128), (int)b);
        const int hrow = (int)(((b * T + c) * H + h) * 64);
#pragma unroll
        for (int nb = 0; nb < S::kNB; ++nb)
            tma_load_2d(sH + buf * S::kHTile + nb * 64 * 128, &tmH, &bars[1 + buf], nb * 64, hrow);
        xh_pending[buf] = xh_issues[buf] & 1;
        xh_issues[buf]++;
    };

    if (tid == 0) {
        mbar_expect_tx(&bars[0], (uint32_t)(S::kCBytes + S::kNB * KJ * 128));
#pragma unroll
        for (int nb = 0; nb < S::kNB; ++nb) {
            tma_load_4d(sC + nb * 128 * 128, &tmC, &bars[0], nb * 64, g, (int)(t0 + row0), (int)b);
            for (int rb = 0; rb <= t; ++rb)
                tma_load_4d(sB + nb * Q * 128 + rb * 128 * 128, &tmB, &bars[0], nb * 64, g,
                            (int)(t0 + rb * 128), (int)b);
        }
        bc_pending = true;
        issue_xh(0);
        if (HG > 1) issue_xh(1);
    }

    // ---- dt of all the CTA's heads over columns [0, KJ) in one coalesced pass
    // (heads of a token are contiguous), then per head the inclusive prefix
    // sum of dt*A in log2 units (warp shuffles).
    for (int e = tid; e < HG * KJ; e += kThreads) {
        const int j = e / HG, k = e - j * HG;
        s_dt[k * Q + j] = (j < len) ? dt[(b * L + t0 + j) * H + head0 + k] : 0.f;
    }
    __syncthreads();
    for (int k = warp; k < HG; k += kThreads / 32) {
        const float Ah = A[head0 + k] * kLog2e;
        float carry = 0.f;
        for (int base = 0; base < KJ; base += 32) {
            float v = s_dt[k * Q + base + lane] * Ah;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            v += carry;
            s_cs[k * Q + base + lane] = v;
            carry = __shfl_sync(0xffffffffu, v, 31);
        }
    }
    __syncthreads();

    // ---- 1. G = C_tile B^T over K = dstate, into TMEM columns [0, KJ).
    if (!mbar_wait(&bars[0], 0, status)) *s_abort = 1;
    __syncthreads();
    bool aborted = *s_abort != 0;
    if (!aborted) {
        if (tid == 0) {
            bc_pending = false;
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, KJ, false, false);
            const uint32_t c0 = smem_u32(sC), b0 = smem_u32(sB);
#pragma unroll
            for (int ks = 0; ks < N / 16; ++ks) {
                const int nb = ks >> 2, ko = (ks & 3) * 32;
                const uint64_t ad = smem_desc_sw128(c0 + nb * 128 * 128 + ko, 16, 1024);
                const uint64_t bd = smem_desc_sw128(b0 + nb * Q * 128 + ko, 16, 1024);
                mma_ss(tmem + kColG, ad, bd, idesc, ks > 0);
            }
            mma_commit(&bars[3]);
            g_pending = 0;
        }
        if (!mbar_wait(&bars[3], 0, status)) *s_abort = 1;
        tc_fence_after();
        __syncthreads();
        aborted = *s_abort != 0;
        if (tid == 0 && !aborted) g_pending = -1;
    }

    const int m = tid;                 // this thread's row within the tile
    const int i = row0 + m;            // ... within the chunk
    const bool row_valid = i < len;

    for (int hi = 0; hi < HG && !aborted; ++hi) {
        const int buf = hi & 1;
        const uint32_t use_parity = (uint32_t)((hi >> 1) & 1);
        const int h = head0 + hi;

        const float* hcs = s_cs + hi * Q;      // this head's prefix sums
        const float* hdt = s_dt + hi * Q;
        const float cs_i = hcs[i];
        float alpha = 0.f;
        if (t > 0) {
            // factorised decay for the block left of the diagonal, through r = cs_{row0 - 1}
            const float r = hcs[row0 - 1];
            s_beta[m] = exp2f(r - hcs[m]) * hdt[m];
            alpha = exp2f(cs_i - r);
        }
        if (!mbar_wait(&bars[1 + buf], use_parity, status)) *s_abort = 1;
        __syncthreads();
        if (*s_abort) { aborted = true; break; }
        if (tid == 0) xh_pending[buf] = -1;

        // ---- 2. decay mask -> TMEM (bf16 pairs), 32 columns at a time
        for (int cb = 0; cb < KJ / 32; ++cb) {
            const int j0 = cb * 32;
            uint32_t packed[16];
            if (j0 >= row0) {
                // diagonal block: exact exponentials, causal mask
                const int rel = (j0 - row0) >> 5;       // column block within the diagonal block
                if (rel > warp) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) packed[q] = 0u;
                } else {
                    uint32_t gr[32];
                    tmem_ld32(tmem + lane_base + kColG + j0, gr);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int ja = j0 + 2 * q, jb = ja + 1;
                        const float va = (ja <= i) ? __uint_as_float(gr[2 * q]) *
                                                         exp2f(cs_i - hcs[ja]) * hdt[ja]
                                                   : 0.f;
                        const float vb = (jb <= i) ? __uint_as_float(gr[2 * q + 1]) *
                                                         exp2f(cs_i - hcs[jb]) * hdt[jb]
                                                   : 0.f;
                        packed[q] = pack_bf16x2(va, vb);
                    }
                }
            } else {
                // block left of the diagonal: G_ij * alpha_i * beta_j
                uint32_t gr[32];
                tmem_ld32(tmem + lane_base + kColG + j0, gr);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int ja = j0 + 2 * q;
                    const float va = __uint_as_float(gr[2 * q]) * alpha * s_beta[ja];
                    const float vb = __uint_as_float(gr[2 * q + 1]) * alpha * s_beta[ja + 1];
                    packed[q] = pack_bf16x2(va, vb);
                }
            }
            tmem_st16(tmem + lane_base + kColM + (uint32_t)(j0 >> 1), packed);
        }
        tc_fence_before();
        __syncthreads();

        // ---- 3. Y = M X (A from TMEM), Z = C_tile h_prev^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idesc_y = idesc_bf16_f32(128, 64, false, true);
            const uint32_t x0 = smem_u32(sX + buf * S::kXTile);
            for (int ks = 0; ks < KJ / 16; ++ks) {
                const uint64_t bd = smem_desc_sw128(x0 + ks * 2048, 16, 1024);
                mma_ts(tmem + kColY, tmem + kColM + ks * 8, bd, idesc_y, ks > 0);
            }
            const uint32_t idesc_z = idesc_bf16_f32(128, 64, false, false);
            const uint32_t c0 = smem_u32(sC), h0 = smem_u32(sH + buf * S::kHTile);
#pragma unroll
            for (int ks = 0; ks < N / 16; ++ks) {
                const int nb = ks >> 2, ko = (ks & 3) * 32;
                const uint64_t ad = smem_desc_sw128(c0 + nb * 128 * 128 + ko, 16, 1024);
                const uint64_t bd = smem_desc_sw128(h0 + nb * 64 * 128 + ko, 16, 1024);
                mma_ss(tmem + kColZ, ad, bd, idesc_z, ks > 0);
            }
            mma_commit(&bars[4]);
            yz_pending = (int)(hi & 1);
        }
        if (!mbar_wait(&bars[4], (uint32_t)(hi & 1), status)) *s_abort = 1;
        tc_fence_after();
        __syncthreads();
        if (*s_abort) { aborted = true; break; }
        if (tid == 0) yz_pending = -1;

        // ---- 4. epilogue: y = Y + exp(cs_i) Z + D_h x, one row per thread
        {
            const float ez = exp2f(cs_i);
            const float Dh = Dv[h];
            const uint8_t* xrow = sX + buf * S::kXTile + i * 128;
            __nv_bfloat16* yrow = y + ((b * L + t0 + i) * H + h) * 64;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t yr[32], zr[32];
                tmem_ld32(tmem + lane_base + kColY + half * 32, yr);
                tmem_ld32(tmem + lane_base + kColZ + half * 32, zr);
                uint32_t out[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    // logical 16-byte chunk (half*4 + q) of the swizzled x row
                    const int lc = half * 4 + q;
                    const uint4 xv = *reinterpret_cast<const uint4*>(xrow + ((lc ^ (i & 7)) << 4));
                    const uint32_t* xu = reinterpret_cast<const uint32_t*>(&xv);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xu[e]));
                        const int k = 8 * q + 2 * e;
                        const float v0 = __uint_as_float(yr[k]) + ez * __uint_as_float(zr[k]) + Dh * xf.x;
                        const float v1 = __uint_as_float(yr[k + 1]) + ez * __uint_as_float(zr[k + 1]) + Dh * xf.y;
                        out[4 * q + e] = pack_bf16x2(v0, v1);
                    }
                }
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(yrow + half * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && hi + 2 < HG) issue_xh(hi + 2);
    }

    if (aborted && tid == 0) {
        if (bc_pending) mbar_wait(&bars[0], 0, status);
        for (int k = 0; k < 2; ++k)
            if (xh_pending[k] >= 0) mbar_wait(&bars[1 + k], (uint32_t)xh_pending[k], status);
        if (g_pending >= 0) mbar_wait(&bars[3], (uint32_t)g_pending, status);
        if (yz_pending >= 0) mbar_wait(&bars[4], (uint32_t)yz_pending, status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

int pick_heads_per_cta(int64_t H, int64_t G) {
    const int64_t hpg = H / G;
    for (int hg = 8; hg > 1; --hg)
        if (hpg % hg == 0) return hg;
    return 1;
}

template <int Q, int N>
cudaError_t launch_impl(const void* x, const float* dt, const float* A, const void* B,
                        const void* C, const float* D, const void* prev, void* y, const Dims& d,
                        cudaStream_t s) {
    using S = OutSmem<Q, N>;
    CUtensorMap tmX, tmB, tmC, tmH;
    const uint64_t xdims[4] = {64, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t xstr[3] = {64 * 2, (uint64_t)(d.H * 64 * 2), (uint64_t)(d.L * d.H * 64 * 2)};
    const uint32_t box128[4] = {64, 1, 128, 1};
    cudaError_t e = make_tmap_bf16(&tmX, x, 4, xdims, xstr, box128);
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
    unsigned int* status = device_status_ptr();
    if (!status) return cudaErrorUnknown;

    const int HG = pick_heads_per_cta(d.H, d.G);
    e = cudaFuncSetAttribute(chunk_out_tc_kernel<Q, N>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(d.b * d.T * (Q / 128)), (unsigned)(d.H / HG));
    chunk_out_tc_kernel<Q, N><<<grid, kThreads, S::kAlloc, s>>>(
        tmX, tmB, tmC, tmH, dt, A, D, static_cast<__nv_bfloat16*>(y), d.L, (int)d.H, (int)d.G,
        d.T, HG, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_out_tc(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, const void* prev, void* y,
                                const Dims& d, cudaStream_t s) {
    if (d.Q == 256 && d.N == 128) return launch_impl<256, 128>(x, dt, A, B, C, D, prev, y, d, s);
    if (d.Q == 256 && d.N == 64) return launch_impl<256, 64>(x, dt, A, B, C, D, prev, y, d, s);
    if (d.Q == 128 && d.N == 128) return launch_impl<128, 128>(x, dt, A, B, C, D, prev, y, d, s);
    if (d.Q == 128 && d.N == 64) return launch_impl<128, 64>(x, dt, A, B, C, D, prev, y, d, s);
    return cudaErrorNotSupported;
}

}  // namespace ssd
