// backward_tc.cu -- the block-decomposed SSD backward on the tcgen05 tensor
// cores (bf16 inputs, fp32 accumulation, fp32 gradients), in chunks of 128
// tokens.  "Transformers are SSMs" (CiteArk), AI research summary: training is
// what the layer is for, and the chunked (block) decomposition that makes the
// forward a set of dense contractions does the same for its gradients.
//
// Per chunk c of a (batch, head), with cs_t the inclusive prefix of dt A over
// the chunk, E_ts = exp(cs_t - cs_s) for s <= t (else 0), el_s = exp(cs_last -
// cs_s), ei_t = exp(cs_t), h the state entering the chunk and Gam = dL/dh of the
// state it hands on (both P x N, from two passes over the chunks run before
// these kernels: the forward's entering states, and the reverse pass
// Gam_{c-1} = exp(cs_last) Gam_c + sum_t ei_t dy_t C_t^T):
//
//   G = C B^T,  R = dy x^T                         (Q x Q, per group / per head)
//   dxpre_s = sum_t G_ts E_ts dy_t + el_s Gam B_s  (P)
//   dx_s    = dt_s dxpre_s + D dy_s
//   dB_s    = sum_h [ sum_t R_ts E_ts dt_s C_t + dt_s el_s Gam^T x_s ]
//   dC_t    = sum_h [ sum_s R_ts E_ts dt_s B_s + ei_t h^T dy_t ]
//   dD      = sum dy . x
// and for the decay: with W_ts = G_ts E_ts dt_s R_ts (fp32),
//   dcs_t = sum_s W_ts - sum_s W_st + ei_t dy_t . (h C_t) - dt_t el_t x_t . (Gam B_t)
//           + [t = last] ( sum_s dt_s el_s x_s . (Gam B_s) + exp(cs_last) <Gam, h> )
//   da_u  = sum_{t >= u} dcs_t,   ddt_u = x_u . dxpre_u + A da_u,   dA = sum dt_u da_u.
// The decay terms are taken from W in fp32 (its row and column sums), not
// from the bf16 operands of the other products: their row and column sums
// cancel to within rounding of each other, and bf16 rounding there would not.
// For the same reason Gam and h enter X1, Ys and <Gam, h> (whose sums nearly
// cancel at a chunk's last token) as bf16 value + residue pairs, near fp32.
// Below the diagonal E factorises through each 32-column block's last column
// r (E_ts = 2^(cs_t - r) 2^(r - cs_s), both <= 1): one exponential a row and
// one a column; the diagonal blocks take one per element.
//
// Two kernels, one CTA per (batch, chunk, group) looping over the group's
// heads, 192 threads: warps 0-3 = the epilogue (thread u = token row u = TMEM
// lane u), warp 4 = TMA producer, warp 5 = MMA issuer (and TMEM owner).  A
// head's inputs come into one of two slots while the previous head computes
// (bwd_dx: x and dy in two slots, Gam and h with their residues in one,
// released once <Gam, h> and the MMAs that read them are done; bwd_dbc: all
// four in two slots).
//   bwd_dx:  G once; per head R, X1 = B Gam^T, Ys = C h^T, then M1 =
//            bf16(G o E) built by the epilogue (with W's row and column
//            sums), then dxi = M1^T dy; the epilogue stages dx in the M1 tile
//            for a TMA store, writes ddt and adds the head's dA and dD.
//   bwd_dbc: per head R, then M2 = bf16(R o E o dt_s) and x, dy scaled in
//            place (dt_s el_s x_s, ei_t dy_t), then dC += M2 B + dy' h and
//            dB += M2^T C + x' Gam accumulated in TMEM over the heads; the
//            epilogue writes dB and dC once.
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

constexpr int kQ = 128;          // tokens per chunk
constexpr int kThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;

// XY: slots for x and dy; GH: slots for Gam and h; kCols: the column-sum
// scratch of W; kLo: Gam and h come with their rounding residues (hi + lo).
template <int N, int XY, int GH, bool kCols, bool kLo>
struct BwdSmem {
    static constexpr int kXY = XY, kGHn = GH;
    static constexpr bool kHasLo = kLo;
    static constexpr int kNB = N / 64;                // 64-column blocks of dstate
    static constexpr int kTok = kQ * 128;             // 128 token rows x 128 B
    static constexpr int kSt = 64 * 128;              // 64 state rows (p) x 128 B
    static constexpr int kGH = kNB * kSt;             // one state tile (Gam or h)
    static constexpr int kC = 0;                      // C tile (kNB blocks)
    static constexpr int kB = kC + kNB * kTok;        // B tile
    static constexpr int kX = kB + kNB * kTok;        // x slots
    static constexpr int kDy = kX + XY * kTok;        // dy slots
    // a Gam/h slot: Gam, [Gam lo], h, [h lo]
    static constexpr int kGHSlot = (kLo ? 4 : 2) * kGH;
    static constexpr int kGHBase = kDy + XY * kTok;
    static constexpr int kGamOff = 0;
    static constexpr int kHpOff = (kLo ? 2 : 1) * kGH;
    static constexpr int gam_lo_off() { return kGH; }
    static constexpr int hp_lo_off() { return 3 * kGH; }
    static constexpr int kM = kGHBase + GH * kGHSlot; // bf16 128 x 128 (two 64-column blocks)
    static constexpr int kCs = kM + 2 * kTok;         // float[128]: cs (log2 units)
    static constexpr int kDt = kCs + kQ * 4;          // float[128]: dt
    static constexpr int kCol = kDt + kQ * 4;         // float[128]: column sums of W
    static constexpr int kRed = kCol + (kCols ? kQ * 4 : 0);       // float[32]: reductions
    static constexpr int kBar = kRed + 32 * 4;
    static constexpr int kTmem = kBar + 16 * 8;
    static constexpr int kCnt = kTmem + 16;           // [0] heads loaded, [1] MMAs issued
    static constexpr int kFlags = kCnt + 16;
    static constexpr int kTotal = kFlags + 16;
    static constexpr int kAlloc = kTotal + 1024;      // slack to align the base to 1 KB
    static_assert(kAlloc <= 232448, "shared memory per CTA");
};
template <int N> using DxSmem = BwdSmem<N, 2, 1, true, true>;
template <int N> using DbcSmem = BwdSmem<N, 2, 2, false, false>;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Column sums of a warp's 32 x 32 block: lane l holds row l in v[0..31]; on
// return v[0] of lane l is the sum of column l over the 32 lanes (a
// reduce-scatter: each step hands half of the remaining columns to the
// partner lane and adds the half it gets back).
__device__ __forceinline__ void warp_column_sums(float (&v)[32], int lane) {
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
        const bool up = (lane & k) != 0;
#pragma unroll
        for (int i = 0; i < k; ++i) {
            const float send = up ? v[i] : v[i + k];
            const float keep = up ? v[i + k] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
        }
    }
}

__device__ __forceinline__ float2 bf2(uint32_t w) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
}

// Inclusive prefix of dt_u A (log2 units) over the chunk's 128 rows (threads
// 0..127, barrier 1); returns cs_u, sets *total to cs of the last row.
__device__ __forceinline__ float chunk_prefix(float a2, int warp, int lane, float* s_red,
                                              float* total) {
    float incl = a2;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_red[warp] = incl;
    named_bar_sync(1, 128);
    float off = 0.f, tot = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const float sw = s_red[w];
        if (w < warp) off += sw;
        tot += sw;
    }
    *total = tot;
    return incl + off;
}

enum {
    BAR_BC = 0,        // C and B tiles loaded
    BAR_XYFULL = 1,    // 2: a slot's x and dy loaded
    BAR_XYEMPTY = 3,   // 2: a slot's x and dy consumed
    BAR_GHFULL = 5,    // 2: a slot's Gam and h loaded
    BAR_GHEMPTY = 7,   // 2: a slot's Gam and h consumed
    BAR_G = 9,         // dx: G computed
    BAR_ACC1 = 10,     // dx: R, X1, Ys computed / dbc: R computed
    BAR_MREADY = 11,   // the epilogue's bf16 operand (and scaled rows) written
    BAR_ACC2 = 12,     // dx: dxi computed
    BAR_ACCEMPTY = 13, // dx: the epilogue has read the head's accumulators
    BAR_DONE = 14,     // dbc: all heads' MMAs completed
    BAR_DRAIN = 15,    // every MMA issued has completed (error path)
    BAR_COUNT = 16
};

// Producer: the C and B tiles of the chunk, then per head x, dy (slot i % XY)
// and Gam, h (and their residues; slot i % GH), each as soon as its slot is free.
template <class S>
__device__ __forceinline__ void produce(uint8_t* smem, uint64_t* bars, const CUtensorMap* tmX,
                                        const CUtensorMap* tmDy, const CUtensorMap* tmB,
                                        const CUtensorMap* tmC, const CUtensorMap* tmGam,
                                        const CUtensorMap* tmHp, const CUtensorMap* tmGamLo,
                                        const CUtensorMap* tmHpLo, int64_t b, int64_t c, int64_t T,
                                        int g, int H, int head0, int nh, volatile int* s_cnt,
                                        volatile int* s_flag, const WaitCtx& status) {
    constexpr int XY = S::kXY, GH = S::kGHn;
    const int t0 = (int)(c * kQ);
    mbar_expect_tx(&bars[BAR_BC], 2 * S::kNB * S::kTok);
    for (int nb = 0; nb < S::kNB; ++nb) {
        tma_load_4d(smem + S::kC + nb * S::kTok, tmC, &bars[BAR_BC], nb * 64, g, t0, (int)b);
        tma_load_4d(smem + S::kB + nb * S::kTok, tmB, &bars[BAR_BC], nb * 64, g, t0, (int)b);
    }
    bool ok = true;
    for (int i = 0; i < nh && ok; ++i) {
        const int hv = head0 + i;
        const int sx = i % XY, sg = i % GH;
        if (i >= XY) ok = mbar_wait(&bars[BAR_XYEMPTY + sx], (uint32_t)((i / XY - 1) & 1), status);
        if (!ok) break;
        mbar_expect_tx(&bars[BAR_XYFULL + sx], 2 * S::kTok);
        tma_load_4d(smem + S::kX + sx * S::kTok, tmX, &bars[BAR_XYFULL + sx], 0, hv, t0, (int)b);
        tma_load_4d(smem + S::kDy + sx * S::kTok, tmDy, &bars[BAR_XYFULL + sx], 0, hv, t0, (int)b);
        if (i >= GH) ok = mbar_wait(&bars[BAR_GHEMPTY + sg], (uint32_t)((i / GH - 1) & 1), status);
        if (!ok) break;
        const int row = (int)(((b * T + c) * H + hv) * 64);
        uint8_t* slot = smem + S::kGHBase + sg * S::kGHSlot;
        mbar_expect_tx(&bars[BAR_GHFULL + sg], S::kGHSlot);
        for (int nb = 0; nb < S::kNB; ++nb) {
            tma_load_2d(slot + S::kGamOff + nb * S::kSt, tmGam, &bars[BAR_GHFULL + sg], nb * 64, row);
            tma_load_2d(slot + S::kHpOff + nb * S::kSt, tmHp, &bars[BAR_GHFULL + sg], nb * 64, row);
            if constexpr (S::kHasLo) {
                tma_load_2d(slot + S::gam_lo_off() + nb * S::kSt, tmGamLo, &bars[BAR_GHFULL + sg],
                            nb * 64, row);
                tma_load_2d(slot + S::hp_lo_off() + nb * S::kSt, tmHpLo, &bars[BAR_GHFULL + sg],
                            nb * 64, row);
            }
        }
        s_cnt[0] = i + 1;
    }
    if (!ok) s_flag[0] = 1;
}

// Error path: before shared memory and TMEM go away, wait (bounded) for the
// loads of the last heads issued and for every MMA issued (the MMA thread
// commits BAR_DRAIN on its way out).
template <class S>
__device__ __forceinline__ void drain(uint64_t* bars, volatile int* s_cnt, const WaitCtx& status) {
    constexpr int XY = S::kXY, GH = S::kGHn;
    mbar_wait(&bars[BAR_BC], 0, status);
    const int nl = s_cnt[0];
    for (int i = (nl > 2 ? nl - 2 : 0); i < nl; ++i) {
        mbar_wait(&bars[BAR_XYFULL + i % XY], (uint32_t)((i / XY) & 1), status);
        mbar_wait(&bars[BAR_GHFULL + i % GH], (uint32_t)((i / GH) & 1), status);
    }
    if (s_cnt[1] > 0) mbar_wait(&bars[BAR_DRAIN], 0, status);
}

__device__ __forceinline__ uint64_t desc(const uint8_t* p, uint32_t lbo) {
    return smem_desc_sw128(smem_u32(p), lbo, 1024);
}

// ============================================================== dx, ddt, dA, dD
template <int N>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dx_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmDy,
                 const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                 const __grid_constant__ CUtensorMap tmGam, const __grid_constant__ CUtensorMap tmHp,
                 const __grid_constant__ CUtensorMap tmGamLo, const __grid_constant__ CUtensorMap tmHpLo,
                 const __grid_constant__ CUtensorMap tmDx,
                 const float* __restrict__ dt, const float* __restrict__ A,
                 const float* __restrict__ Dv, float* __restrict__ ddt,
                 float* __restrict__ dA, float* __restrict__ dD, int64_t L, int H, int G,
                 int64_t T, int ksplit, int pcols, WaitCtx status) {
    // H counts virtual heads (headdim 64); real head = virtual head / ksplit
    using S = DxSmem<N>;
    constexpr uint32_t kColG = 0, kColR = 128, kColDx = 256, kColX1 = 320, kColYs = 384;
    constexpr uint32_t kTmemCols = 512;
    const int Hr = H / ksplit;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = (int)(blockIdx.x % G);
    const int64_t bc = blockIdx.x / G;
    const int64_t c = bc % T, b = bc / T;
    const int64_t t0 = c * kQ;
    const int nh = H / G, head0 = g * nh;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sC = smem + S::kC;
    uint8_t* sB = smem + S::kB;
    uint8_t* sGam = smem + S::kGHBase + S::kGamOff;     // one Gam/h slot
    uint8_t* sGamLo = smem + S::kGHBase + S::gam_lo_off();
    uint8_t* sHp = smem + S::kGHBase + S::kHpOff;
    uint8_t* sHpLo = smem + S::kGHBase + S::hp_lo_off();
    uint8_t* sM = smem + S::kM;
    float* s_cs = reinterpret_cast<float*>(smem + S::kCs);
    float* s_dt = reinterpret_cast<float*>(smem + S::kDt);
    float* s_col = reinterpret_cast<float*>(smem + S::kCol);
    float* s_red = reinterpret_cast<float*>(smem + S::kRed);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_cnt = reinterpret_cast<volatile int*>(smem + S::kCnt);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + S::kFlags);

    if (tid == 0) {
        for (int i = 0; i < BAR_COUNT; ++i) mbar_init(&bars[i], 1);
        s_cnt[0] = 0;
        s_cnt[1] = 0;
        s_flag[0] = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 4) {
        // ================================================== TMA producer
        if (lane == 0)
            produce<S>(smem, bars, &tmX, &tmDy, &tmB, &tmC, &tmGam, &tmHp, &tmGamLo, &tmHpLo, b, c,
                       T, g, H, head0, nh, s_cnt, s_flag, status);
    } else if (warp == 5) {
        // ================================================== MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait(&bars[BAR_BC], 0, status);
            if (ok) {
                tc_fence_after();
                // G = C B^T (M = t, N = s, K = n), both K-major
                const uint32_t idG = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
                for (int ks = 0; ks < N / 16; ++ks) {
                    const int ko = (ks >> 2) * S::kTok + (ks & 3) * 32;
                    mma_ss(tmem + kColG, desc(sC + ko, 16), desc(sB + ko, 16), idG, ks > 0);
                }
                mma_commit(&bars[BAR_G]);
                s_cnt[1] = 1;
            }
            const uint32_t idR = idesc_bf16_f32(128, 128, false, false);   // dy, x K-major
            const uint32_t idS = idesc_bf16_f32(128, 64, false, false);    // B|C, Gam|h K-major
            const uint32_t idD = idesc_bf16_f32(128, 64, true, true);      // M1, dy MN-major
            for (int i = 0; i < nh && ok; ++i) {
                const int sx = i % S::kXY;
                ok = mbar_wait(&bars[BAR_XYFULL + sx], (uint32_t)((i / S::kXY) & 1), status) &&
                     mbar_wait(&bars[BAR_GHFULL], (uint32_t)(i & 1), status) &&
                     (i == 0 || mbar_wait(&bars[BAR_ACCEMPTY], (uint32_t)((i - 1) & 1), status));
                if (!ok) break;
                tc_fence_after();
                const uint8_t* sX = smem + S::kX + sx * S::kTok;
                const uint8_t* sDy = smem + S::kDy + sx * S::kTok;
                // R = dy x^T (M = t, N = s, K = p)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + kColR, desc(sDy + ks * 32, 16), desc(sX + ks * 32, 16), idR, ks > 0);
                // X1 = B Gam^T (M = s, N = p, K = n); Ys = C h^T (M = t, N = p, K = n);
                // Gam and h as hi + lo (their bf16 rounding residue), so these
                // two products, whose sums cancel in the decay gradient, carry
                // Gam and h to near fp32
#pragma unroll
                for (int ks = 0; ks < N / 16; ++ks) {
                    const int ko = (ks >> 2) * S::kTok + (ks & 3) * 32;
                    const int so = (ks >> 2) * S::kSt + (ks & 3) * 32;
                    mma_ss(tmem + kColX1, desc(sB + ko, 16), desc(sGam + so, 16), idS, ks > 0);
                    mma_ss(tmem + kColYs, desc(sC + ko, 16), desc(sHp + so, 16), idS, ks > 0);
                }
#pragma unroll
                for (int ks = 0; ks < N / 16; ++ks) {
                    const int ko = (ks >> 2) * S::kTok + (ks & 3) * 32;
                    const int so = (ks >> 2) * S::kSt + (ks & 3) * 32;
                    mma_ss(tmem + kColX1, desc(sB + ko, 16), desc(sGamLo + so, 16), idS, true);
                    mma_ss(tmem + kColYs, desc(sC + ko, 16), desc(sHpLo + so, 16), idS, true);
                }
                mma_commit(&bars[BAR_ACC1]);
                ok = mbar_wait(&bars[BAR_MREADY], (uint32_t)(i & 1), status);
                if (!ok) break;
                tc_fence_after();
                // dxi = M1^T dy (M = s, N = p, K = t): M1 as stored (rows t, s
                // contiguous) is MN-major, its two 64-column blocks 16 KB apart
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss(tmem + kColDx, desc(sM + ks * 2048, S::kTok), desc(sDy + ks * 2048, 16),
                           idD, ks > 0);
                mma_commit(&bars[BAR_ACC2]);
            }
            if (s_cnt[1]) mma_commit(&bars[BAR_DRAIN]);
            if (!ok) s_flag[0] = 1;
        }
    } else {
        // ================================================== epilogue (warps 0-3)
        const int u = tid;
        const uint32_t lb = (uint32_t)(warp * 32) << 16;
        const bool row_in = t0 + u < L;
        const float* dt_row = dt + (b * L + t0 + u) * Hr;
        bool fail = false;
        float ddt_acc = 0.f, dA_acc = 0.f, dD_acc = 0.f;
        float dt_next = (row_in && nh > 0) ? dt_row[head0 / ksplit] : 0.f;
        s_col[u] = 0.f;   // column sums of W: added to by the warps, read and cleared by thread u
        for (int i = 0; i < nh; ++i) {
            const int hv = head0 + i, hr = hv / ksplit;
            const float Ah = A[hr];
            const float dtu = dt_next;
            if (i + 1 < nh) dt_next = row_in ? dt_row[(hv + 1) / ksplit] : 0.f;
            float csL;
            const float csu = chunk_prefix(dtu * Ah * kLog2e, warp, lane, s_red, &csL);
            s_cs[u] = csu;
            s_dt[u] = dtu;
            if (i == 0) fail = fail || !mbar_wait(&bars[BAR_G], 0, status);
            fail = fail || !mbar_wait(&bars[BAR_ACC1], (uint32_t)(i & 1), status);
            // the M1 tile is rewritten below: the previous head's dx store must
            // have read it
            if (u == 0) bulk_wait_group_read<0>();
            if (named_bar_or(2, 128, fail)) {   // also publishes s_cs, s_dt
                fail = true;
                break;
            }
            tc_fence_after();
            // ---- <Gam, h> over this thread's share (the tiles share one layout),
            // each as hi + lo
            float zp = 0.f;
            {
                const uint4* g4 = reinterpret_cast<const uint4*>(sGam);
                const uint4* gl4 = reinterpret_cast<const uint4*>(sGamLo);
                const uint4* h4 = reinterpret_cast<const uint4*>(sHp);
                const uint4* hl4 = reinterpret_cast<const uint4*>(sHpLo);
#pragma unroll 2
                for (int k = 0; k < S::kGH / 16 / 128; ++k) {
                    const uint4 gv = g4[u + 128 * k], hv4 = h4[u + 128 * k];
                    const uint4 glv = gl4[u + 128 * k], hlv = hl4[u + 128 * k];
                    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
                    const uint32_t hw[4] = {hv4.x, hv4.y, hv4.z, hv4.w};
                    const uint32_t glw[4] = {glv.x, glv.y, glv.z, glv.w};
                    const uint32_t hlw[4] = {hlv.x, hlv.y, hlv.z, hlv.w};
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 a = bf2(gw[e2]), al = bf2(glw[e2]);
                        const float2 bb = bf2(hw[e2]), bl = bf2(hlw[e2]);
                        zp = fmaf(a.x + al.x, bb.x + bl.x, fmaf(a.y + al.y, bb.y + bl.y, zp));
                    }
                }
            }
            // ---- M1 = bf16(G o E) (row u), W = G o E o dt_s o R: row sum, column sums
            float rowsum = 0.f;
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                uint4* mrow = reinterpret_cast<uint4*>(sM + (j >> 1) * S::kTok + u * 128);
                if (j > warp) {
                    // columns s = 32 j .. 32 j + 31 all lie past every row of this warp
#pragma unroll
                    for (int q = 0; q < 4; ++q) mrow[((j & 1) * 4 + q) ^ (u & 7)] = make_uint4(0, 0, 0, 0);
                    continue;
                }
                uint32_t gr[32], rr[32];
                tmem_ld32x2(tmem + lb + kColG + 32 * j, tmem + lb + kColR + 32 * j, gr, rr);
                float v[32];
                uint32_t pk[16];
                if (j < warp) {
                    // a block wholly below the diagonal: the decay factorises
                    // through the block's last column r, 2^(cs_u - cs_s) =
                    // 2^(cs_u - r) 2^(r - cs_s) (both <= 1), one exponential a
                    // row; lane l computes column 32 j + l's factor and the
                    // others take it by shuffle
                    const float r = s_cs[32 * j + 31];
                    const float a = fast_exp2(csu - r);
                    const float bl = fast_exp2(r - s_cs[32 * j + lane]);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int s0 = 32 * j + e;
                        const float m0 = __uint_as_float(gr[e]) * a * __shfl_sync(0xffffffffu, bl, e);
                        const float m1 = __uint_as_float(gr[e + 1]) * a * __shfl_sync(0xffffffffu, bl, e + 1);
                        pk[e >> 1] = pack_bf16x2(m0, m1);
                        v[e] = m0 * s_dt[s0] * __uint_as_float(rr[e]);
                        v[e + 1] = m1 * s_dt[s0 + 1] * __uint_as_float(rr[e + 1]);
                        rowsum += v[e] + v[e + 1];
                    }
                } else {
                    // the diagonal block: an exponential per element, the mask by
                    // selects (no branch per element, so the loads and
                    // exponentials overlap; past the diagonal the exponential
                    // may overflow, and is never selected)
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int s0 = 32 * j + e;
                        const float e0 = __uint_as_float(gr[e]) * fast_exp2(csu - s_cs[s0]);
                        const float e1 = __uint_as_float(gr[e + 1]) * fast_exp2(csu - s_cs[s0 + 1]);
                        const float m0 = s0 <= u ? e0 : 0.f, m1 = s0 + 1 <= u ? e1 : 0.f;
                        pk[e >> 1] = pack_bf16x2(m0, m1);
                        v[e] = m0 * s_dt[s0] * __uint_as_float(rr[e]);
                        v[e + 1] = m1 * s_dt[s0 + 1] * __uint_as_float(rr[e + 1]);
                        rowsum += v[e] + v[e + 1];
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    mrow[((j & 1) * 4 + q) ^ (u & 7)] =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                warp_column_sums(v, lane);
                atomicAdd(&s_col[32 * j + lane], v[0]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, 128);
            if (u == 0) {
                mbar_arrive(&bars[BAR_MREADY]);
                mbar_arrive(&bars[BAR_GHEMPTY]);   // Gam, h: read by their MMAs and above
            }
            float dcs = rowsum - s_col[u];
            s_col[u] = 0.f;   // the next head's additions come after more barriers

            // ---- dx, and the row's dot products
            fail = !mbar_wait(&bars[BAR_ACC2], (uint32_t)(i & 1), status);
            if (named_bar_or(2, 128, fail)) {
                fail = true;
                break;
            }
            tc_fence_after();
            const float el = fast_exp2(csL - csu), ei = fast_exp2(csu);
            const float Dh = Dv[hr];
            float dexpl = 0.f, sU = 0.f, dyys = 0.f, dxd = 0.f;
            const int sx = i % S::kXY;
            const uint4* xrow = reinterpret_cast<const uint4*>(smem + S::kX + sx * S::kTok + u * 128);
            const uint4* dyrow = reinterpret_cast<const uint4*>(smem + S::kDy + sx * S::kTok + u * 128);
            // dx rows are staged in the M1 tile (free once the M1^T dy MMAs
            // are done) as 32-column fp32 boxes, 128-byte swizzled, then stored
            // by TMA (rows past the sequence end clipped by the tensor map)
#pragma unroll 1
            for (int k = 0; k < 2; ++k) {
                uint32_t dr[32], xr1[32], yr[32];
                tmem_ld32x2(tmem + lb + kColDx + 32 * k, tmem + lb + kColX1 + 32 * k, dr, xr1);
                tmem_ld32(tmem + lb + kColYs + 32 * k, yr);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 xv = xrow[(4 * k + q) ^ (u & 7)];
                    const uint4 yv = dyrow[(4 * k + q) ^ (u & 7)];
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                    const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
                    float o[8];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 xf = bf2(xw[e2]), yf = bf2(yw[e2]);
                        const float xe[2] = {xf.x, xf.y}, ye[2] = {yf.x, yf.y};
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const int p = 8 * q + 2 * e2 + h2;
                            const float x1 = __uint_as_float(xr1[p]);
                            const float dxpre = __uint_as_float(dr[p]) + el * x1;
                            o[2 * e2 + h2] = dtu * dxpre + Dh * ye[h2];
                            dexpl += xe[h2] * dxpre;
                            sU += xe[h2] * x1;
                            dyys += ye[h2] * __uint_as_float(yr[p]);
                            dxd += ye[h2] * xe[h2];
                        }
                    }
                    float4* box = reinterpret_cast<float4*>(sM + k * S::kTok + u * 128);
                    box[(2 * q) ^ (u & 7)] = make_float4(o[0], o[1], o[2], o[3]);
                    box[(2 * q + 1) ^ (u & 7)] = make_float4(o[4], o[5], o[6], o[7]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            const float Uu = dtu * el * sU;
            dcs += ei * dyys - Uu;
            {
                const float wu = warp_sum(Uu), wz = warp_sum(zp);
                if (lane == 0) {
                    s_red[4 + warp] = wu;
                    s_red[8 + warp] = wz;
                }
            }
            named_bar_sync(1, 128);   // every read of the head's TMEM, x and dy is done
            if (u == 0) {
                mbar_arrive(&bars[BAR_ACCEMPTY]);
                mbar_arrive(&bars[BAR_XYEMPTY + sx]);
                for (int k = 0; k < pcols / 32; ++k)
                    tma_store_4d(&tmDx, sM + k * S::kTok, 32 * k, hv, (int)t0, (int)b);
                bulk_commit_group();
            }
            if (u == kQ - 1) {
                const float sumU = s_red[4] + s_red[5] + s_red[6] + s_red[7];
                const float sumZ = s_red[8] + s_red[9] + s_red[10] + s_red[11];
                dcs += sumU + fast_exp2(csL) * sumZ;
            }
            // da_u = sum_{t >= u} dcs_t
            float suf = dcs;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += v;
            }
            if (lane == 0) s_red[12 + warp] = suf;
            named_bar_sync(1, 128);
            float da = suf;
            for (int w = warp + 1; w < 4; ++w) da += s_red[12 + w];
            ddt_acc += dexpl + Ah * da;
            dA_acc += dtu * da;
            dD_acc += dxd;
            if (hv % ksplit == ksplit - 1) {
                // the last virtual head of real head hr: write its ddt, add its dA, dD
                if (row_in) ddt[(b * L + t0 + u) * Hr + hr] = ddt_acc;
                const float wa = warp_sum(dA_acc), wd = warp_sum(dD_acc);
                if (lane == 0) {
                    s_red[16 + warp] = wa;
                    s_red[20 + warp] = wd;
                }
                named_bar_sync(1, 128);
                if (u == 0) {
                    atomicAdd(dA + hr, s_red[16] + s_red[17] + s_red[18] + s_red[19]);
                    atomicAdd(dD + hr, s_red[20] + s_red[21] + s_red[22] + s_red[23]);
                }
                ddt_acc = dA_acc = dD_acc = 0.f;
            }
        }
        if (u == 0) bulk_wait_group<0>();      // dx stores done before the CTA leaves
        if (fail) s_flag[0] = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (s_flag[0] && tid == 4 * 32) drain<S>(bars, s_cnt, status);
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ============================================================== dB, dC
template <int N>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dbc_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmDy,
                  const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                  const __grid_constant__ CUtensorMap tmGam, const __grid_constant__ CUtensorMap tmHp,
                  const float* __restrict__ dt, const float* __restrict__ A,
                  float* __restrict__ dB, float* __restrict__ dC, int64_t L, int H, int G,
                  int64_t T, int ksplit, WaitCtx status) {
    using S = DbcSmem<N>;
    constexpr uint32_t kColR = 0, kColDC = 128, kColDB = 128 + N;
    constexpr uint32_t kTmemCols = (N == 128) ? 512 : 256;
    const int Hr = H / ksplit;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = (int)(blockIdx.x % G);
    const int64_t bc = blockIdx.x / G;
    const int64_t c = bc % T, b = bc / T;
    const int64_t t0 = c * kQ;
    const int nh = H / G, head0 = g * nh;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sC = smem + S::kC;
    uint8_t* sB = smem + S::kB;
    uint8_t* sM = smem + S::kM;
    float* s_cs = reinterpret_cast<float*>(smem + S::kCs);
    float* s_dt = reinterpret_cast<float*>(smem + S::kDt);
    float* s_red = reinterpret_cast<float*>(smem + S::kRed);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_cnt = reinterpret_cast<volatile int*>(smem + S::kCnt);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + S::kFlags);

    if (tid == 0) {
        for (int i = 0; i < BAR_COUNT; ++i) mbar_init(&bars[i], 1);
        s_cnt[0] = 0;
        s_cnt[1] = 0;
        s_flag[0] = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 4) {
        if (lane == 0)
            produce<S>(smem, bars, &tmX, &tmDy, &tmB, &tmC, &tmGam, &tmHp, nullptr, nullptr, b, c,
                       T, g, H, head0, nh, s_cnt, s_flag, status);
    } else if (warp == 5) {
        if (lane == 0) {
            bool ok = mbar_wait(&bars[BAR_BC], 0, status);
            const uint32_t idR = idesc_bf16_f32(128, 128, false, false);   // dy, x K-major
            const uint32_t idC = idesc_bf16_f32(128, N, false, true);      // M2 | dy' K-major; B | h MN-major
            const uint32_t idB = idesc_bf16_f32(128, N, true, true);       // M2^T MN-major; C MN-major
            const uint32_t idB2 = idesc_bf16_f32(128, N, false, true);     // x' K-major; Gam MN-major
            for (int i = 0; i < nh && ok; ++i) {
                const int sl = i & 1;
                const uint32_t par = (uint32_t)((i >> 1) & 1);
                ok = mbar_wait(&bars[BAR_XYFULL + sl], par, status) &&
                     mbar_wait(&bars[BAR_GHFULL + sl], par, status);
                if (!ok) break;
                tc_fence_after();
                const uint8_t* sX = smem + S::kX + sl * S::kTok;
                const uint8_t* sDy = smem + S::kDy + sl * S::kTok;
                const uint8_t* sGam = smem + S::kGHBase + sl * S::kGHSlot + S::kGamOff;
                const uint8_t* sHp = smem + S::kGHBase + sl * S::kGHSlot + S::kHpOff;
                // R = dy x^T (the previous head's R was read before its MREADY)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + kColR, desc(sDy + ks * 32, 16), desc(sX + ks * 32, 16), idR, ks > 0);
                mma_commit(&bars[BAR_ACC1]);
                s_cnt[1] = 1;
                ok = mbar_wait(&bars[BAR_MREADY], (uint32_t)(i & 1), status);
                if (!ok) break;
                tc_fence_after();
                // dC += M2 B (M = t, N = n, K = s); dC += dy' h (K = p)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss(tmem + kColDC, desc(sM + (ks >> 2) * S::kTok + (ks & 3) * 32, 16),
                           desc(sB + ks * 2048, S::kTok), idC, i > 0 || ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + kColDC, desc(sDy + ks * 32, 16), desc(sHp + ks * 2048, S::kSt), idC,
                           true);
                // dB += M2^T C (M = s, N = n, K = t); dB += x' Gam (K = p)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss(tmem + kColDB, desc(sM + ks * 2048, S::kTok), desc(sC + ks * 2048, S::kTok),
                           idB, i > 0 || ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + kColDB, desc(sX + ks * 32, 16), desc(sGam + ks * 2048, S::kSt), idB2,
                           true);
                mma_commit(&bars[BAR_XYEMPTY + sl]);
                mma_commit(&bars[BAR_GHEMPTY + sl]);
            }
            if (ok) mma_commit(&bars[BAR_DONE]);
            if (s_cnt[1]) mma_commit(&bars[BAR_DRAIN]);
            if (!ok) s_flag[0] = 1;
        }
    } else {
        const int u = tid;
        const uint32_t lb = (uint32_t)(warp * 32) << 16;
        const bool row_in = t0 + u < L;
        const float* dt_row = dt + (b * L + t0 + u) * Hr;
        bool fail = false;
        float dt_next = (row_in && nh > 0) ? dt_row[head0 / ksplit] : 0.f;
        for (int i = 0; i < nh; ++i) {
            const int hv = head0 + i, hr = hv / ksplit;
            const float dtu = dt_next;
            if (i + 1 < nh) dt_next = row_in ? dt_row[(hv + 1) / ksplit] : 0.f;
            float csL;
            const float csu = chunk_prefix(dtu * A[hr] * kLog2e, warp, lane, s_red, &csL);
            s_cs[u] = csu;
            s_dt[u] = dtu;
            fail = !mbar_wait(&bars[BAR_ACC1], (uint32_t)(i & 1), status);
            if (named_bar_or(2, 128, fail)) {   // also publishes s_cs, s_dt
                fail = true;
                break;
            }
            tc_fence_after();
            // ---- M2 = bf16(R o E o dt_s) (row u); R(i) completing implies the
            // previous head's MMAs, the last readers of M2, have completed
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                uint4* mrow = reinterpret_cast<uint4*>(sM + (j >> 1) * S::kTok + u * 128);
                if (j > warp) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) mrow[((j & 1) * 4 + q) ^ (u & 7)] = make_uint4(0, 0, 0, 0);
                    continue;
                }
                uint32_t rr[32];
                tmem_ld32(tmem + lb + kColR + 32 * j, rr);
                uint32_t pk[16];
                if (j < warp) {
                    // as in the dx kernel: below the diagonal, the decay through
                    // the block's last column (one exponential a row, column
                    // factors times dt by shuffle)
                    const float r = s_cs[32 * j + 31];
                    const float a = fast_exp2(csu - r);
                    const float bl = fast_exp2(r - s_cs[32 * j + lane]) * s_dt[32 * j + lane];
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        pk[e >> 1] = pack_bf16x2(
                            __uint_as_float(rr[e]) * a * __shfl_sync(0xffffffffu, bl, e),
                            __uint_as_float(rr[e + 1]) * a * __shfl_sync(0xffffffffu, bl, e + 1));
                } else {
                    // the diagonal block, as in the dx kernel: an exponential per
                    // element, the mask by selects
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int s0 = 32 * j + e;
                        const float e0 = __uint_as_float(rr[e]) * fast_exp2(csu - s_cs[s0]) * s_dt[s0];
                        const float e1 = __uint_as_float(rr[e + 1]) * fast_exp2(csu - s_cs[s0 + 1]) * s_dt[s0 + 1];
                        pk[e >> 1] = pack_bf16x2(s0 <= u ? e0 : 0.f, s0 + 1 <= u ? e1 : 0.f);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    mrow[((j & 1) * 4 + q) ^ (u & 7)] =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
            // ---- x row *= dt_u el_u, dy row *= ei_u, in place (R has consumed them)
            {
                const float sx = dtu * fast_exp2(csL - csu), sy = fast_exp2(csu);
                uint4* xrow = reinterpret_cast<uint4*>(smem + S::kX + (i & 1) * S::kTok + u * 128);
                uint4* yrow = reinterpret_cast<uint4*>(smem + S::kDy + (i & 1) * S::kTok + u * 128);
#pragma unroll
                for (int q0 = 0; q0 < 8; ++q0) {
                    // the row's 16-byte chunks in a rotated order: the lanes of a
                    // phase (rows 128 bytes apart) then hit different banks
                    const int q = q0 ^ (u & 7);
                    uint4 xv = xrow[q], yv = yrow[q];
                    uint32_t* xw = reinterpret_cast<uint32_t*>(&xv);
                    uint32_t* yw = reinterpret_cast<uint32_t*>(&yv);
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 xf = bf2(xw[e2]), yf = bf2(yw[e2]);
                        xw[e2] = pack_bf16x2(xf.x * sx, xf.y * sx);
                        yw[e2] = pack_bf16x2(yf.x * sy, yf.y * sy);
                    }
                    xrow[q] = xv;
                    yrow[q] = yv;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, 128);
            if (u == 0) mbar_arrive(&bars[BAR_MREADY]);
        }
        // ---- dC and dB rows out (fp32)
        if (!fail) {
            fail = !mbar_wait(&bars[BAR_DONE], 0, status);
            fail = named_bar_or(2, 128, fail);
        }
        if (!fail) {
            tc_fence_after();
            float* dco = dC + ((b * L + t0 + u) * G + g) * (int64_t)N;
            float* dbo = dB + ((b * L + t0 + u) * G + g) * (int64_t)N;
#pragma unroll 1
            for (int k = 0; k < N / 32; ++k) {
                uint32_t cr[32], br[32];
                tmem_ld32x2(tmem + lb + kColDC + 32 * k, tmem + lb + kColDB + 32 * k, cr, br);
                if (row_in) {
                    float4* c4 = reinterpret_cast<float4*>(dco + 32 * k);
                    float4* b4 = reinterpret_cast<float4*>(dbo + 32 * k);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        c4[q] = make_float4(__uint_as_float(cr[4 * q]), __uint_as_float(cr[4 * q + 1]),
                                            __uint_as_float(cr[4 * q + 2]), __uint_as_float(cr[4 * q + 3]));
                        b4[q] = make_float4(__uint_as_float(br[4 * q]), __uint_as_float(br[4 * q + 1]),
                                            __uint_as_float(br[4 * q + 2]), __uint_as_float(br[4 * q + 3]));
                    }
                }
            }
            tc_fence_before();
        }
        if (fail) s_flag[0] = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (s_flag[0] && tid == 4 * 32) drain<S>(bars, s_cnt, status);
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int N>
cudaError_t launch_impl(const void* x, const void* dy, const float* dt, const float* A,
                        const void* B, const void* C, const float* D, const void* hp,
                        const void* hp_lo, const void* gam, const void* gam_lo, float* dx,
                        float* ddt, float* dA, float* dB, float* dC, float* dD, const Dims& d,
                        int ksplit, int pc, cudaStream_t s) {
    CUtensorMap tmX, tmDy, tmB, tmC, tmGam, tmHp, tmGamLo, tmHpLo;
    // x and dy: pc columns a (virtual) head; a 64-column box reads zeros past them
    const uint64_t xdims[4] = {(uint64_t)pc, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t xstr[3] = {(uint64_t)pc * 2, (uint64_t)(d.H * pc * 2), (uint64_t)(d.L * d.H * pc * 2)};
    const uint32_t box128[4] = {64, 1, kQ, 1};
    cudaError_t e = make_tmap_bf16(&tmX, x, 4, xdims, xstr, box128);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&tmDy, dy, 4, xdims, xstr, box128);
    if (e != cudaSuccess) return e;
    const uint64_t bdims[4] = {(uint64_t)N, (uint64_t)d.G, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t bstr[3] = {(uint64_t)N * 2, (uint64_t)(d.G * N * 2), (uint64_t)(d.L * d.G * N * 2)};
    e = make_tmap_bf16(&tmB, B, 4, bdims, bstr, box128);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&tmC, C, 4, bdims, bstr, box128);
    if (e != cudaSuccess) return e;
    // per-chunk states: rows (b, T, H, 64) of N bf16
    const uint64_t hdims[2] = {(uint64_t)N, (uint64_t)(d.b * d.T * d.H * 64)};
    const uint64_t hstr[1] = {(uint64_t)N * 2};
    const uint32_t hbox[2] = {64, 64};
    const void* planes[4] = {gam, hp, gam_lo, hp_lo};
    CUtensorMap* maps[4] = {&tmGam, &tmHp, &tmGamLo, &tmHpLo};
    for (int k = 0; k < 4; ++k) {
        e = make_tmap_bf16(maps[k], planes[k], 2, hdims, hstr, hbox);
        if (e != cudaSuccess) return e;
    }
    // dx (b, L, H, pc) fp32 as 32-column boxes of 128 rows, 128-byte swizzled
    CUtensorMap tmDx;
    {
        const uint64_t ddims[4] = {(uint64_t)pc, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
        const uint64_t dstr[3] = {(uint64_t)pc * 4, (uint64_t)(d.H * pc * 4), (uint64_t)(d.L * d.H * pc * 4)};
        const uint32_t dbox[4] = {32, 1, kQ, 1};
        e = make_tmap_f32_plain(&tmDx, dx, 4, ddims, dstr, dbox, true);
        if (e != cudaSuccess) return e;
    }
    const sm100::WaitCtx status = make_wait_ctx();
    if (!status.word) return cudaErrorUnknown;

    const int64_t grid = d.b * d.T * d.G;
    if (grid == 0) return cudaSuccess;
    e = cudaFuncSetAttribute(bwd_dx_tc_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DxSmem<N>::kAlloc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_dbc_tc_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DbcSmem<N>::kAlloc);
    if (e != cudaSuccess) return e;
    bwd_dx_tc_kernel<N><<<(unsigned)grid, kThreads, DxSmem<N>::kAlloc, s>>>(
        tmX, tmDy, tmB, tmC, tmGam, tmHp, tmGamLo, tmHpLo, tmDx, dt, A, D, ddt, dA, dD, d.L,
        (int)d.H, (int)d.G, d.T, ksplit, pc, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_dbc_tc_kernel<N><<<(unsigned)grid, kThreads, DbcSmem<N>::kAlloc, s>>>(
        tmX, tmDy, tmB, tmC, tmGam, tmHp, dt, A, dB, dC, d.L, (int)d.H, (int)d.G, d.T, ksplit,
        status);
    return cudaGetLastError();
}

// Workspace carve-up of the tensor-core backward (Q = 128 chunks): the
// entering states and dL/dh per chunk, each as bf16 hi and lo planes; one
// fp32 buffer of chunk states (forward, then reverse); the log-decays.
struct BwdLayout {
    size_t prev = 0, prev_lo = 0, gam = 0, gam_lo = 0, states = 0, logdecay = 0, total = 0;
};
BwdLayout bwd_layout(const Dims& q) {
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t elems = (size_t)(q.b * q.T * q.H * state_rows(q.P) * q.N);
    BwdLayout w;
    w.prev = 0;
    w.prev_lo = up(w.prev + elems * 2);
    w.gam = up(w.prev_lo + elems * 2);
    w.gam_lo = up(w.gam + elems * 2);
    w.states = up(w.gam_lo + elems * 2);
    w.logdecay = up(w.states + elems * 4);
    w.total = up(w.logdecay + (size_t)(q.b * q.T * q.H) * 4);
    return w;
}

Dims chunks128(const Dims& d) {
    Dims q = d;
    q.Q = kQ;
    q.T = (d.L + kQ - 1) / kQ;
    return q;
}

}  // namespace

bool backward_tc_supported(const Dims& d, Elt t) { return tc_supported(chunks128(d), t); }

size_t backward_tc_workspace_bytes(const Dims& d) { return bwd_layout(chunks128(d)).total; }

cudaError_t launch_backward_tc(const void* x, const float* dt, const float* A, const void* B,
                               const void* C, const float* D, const float* init, const void* dy,
                               const float* dfinal, float* dx, float* ddt, float* dA, float* dB,
                               float* dC, float* dD, float* dinit, void* ws, const Dims& d,
                               cudaStream_t s) {
    const Dims q = chunks128(d);
    Dims qs = q;                          // the state buffers' rows a head
    qs.P = state_rows(d.P);
    const BwdLayout w = bwd_layout(q);
    char* base = static_cast<char*>(ws);
    void* prev = base + w.prev;
    void* prev_lo = base + w.prev_lo;
    void* gam = base + w.gam;
    void* gam_lo = base + w.gam_lo;
    float* states = reinterpret_cast<float*>(base + w.states);
    float* logdecay = reinterpret_cast<float*>(base + w.logdecay);
    // the states entering each chunk (the forward's, recomputed), hi + lo
    cudaError_t e = launch_chunk_state_tc(x, dt, A, B, states, logdecay, q, s);
    if (e != cudaSuccess) return e;
    e = launch_state_pass(states, logdecay, init, prev, nullptr, qs, Elt::BF16, s, false, d.P,
                          prev_lo);
    if (e != cudaSuccess) return e;
    // dL/dh of the state each chunk hands on (hi + lo), and dL/dinit
    e = launch_chunk_state_tc(dy, dt, A, C, states, logdecay, q, s, true);
    if (e != cudaSuccess) return e;
    e = launch_state_pass(states, logdecay, dfinal, gam, dinit, qs, Elt::BF16, s, true, d.P,
                          gam_lo);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(dA, 0, sizeof(float) * (size_t)d.H, s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(dD, 0, sizeof(float) * (size_t)d.H, s);
    if (e != cudaSuccess) return e;
    int k = 1;
    const Dims v = virtual_heads(q, &k);
    if (v.N == 128)
        return launch_impl<128>(x, dy, dt, A, B, C, D, prev, prev_lo, gam, gam_lo, dx, ddt, dA, dB,
                                dC, dD, v, k, head_cols(d), s);
    if (v.N == 64)
        return launch_impl<64>(x, dy, dt, A, B, C, D, prev, prev_lo, gam, gam_lo, dx, ddt, dA, dB,
                               dC, dD, v, k, head_cols(d), s);
    return cudaErrorNotSupported;
}

}  // namespace ssd
