// chunk_out_body.cuh -- one tile of the chunk outputs on the tcgen05 tensor
// cores (bf16 inputs, fp32 accumulation): steps a1 + a4 of the
// block-decomposed SSD forward.  Used by the output kernel (chunk_out_tc.cu)
// and by the output role of the fused walk + output kernel.
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
// A tile is (batch, chunk, 128-row tile t of the chunk, group of HG heads
// sharing B and C), one CTA's work.  Heads are virtual heads of headdim 64: a head of
// headdim 64 k is k of them, sharing dt, A and D.  Tile t holds rows i in [128 t, 128 t + 128).
//
// The decay between row i and column j < i factorises through any boundary r:
// exp(cs_i - cs_j) = exp(cs_i - r) exp(r - cs_j).  The diagonal 128 x 128
// block, Y_i = sum_{j <= i} G_ij exp(cs_i - cs_j) dt_j x_j, factorises through
// one boundary r1 for the whole tile: with
//   a_i = 2^(cs_i - r1),  b_j = 2^(r1 - cs_j) dt_j   (cs in log2 units),
//   Y = diag(a) (G o causal) (b * X_t),
// so the bf16 operand G o causal is built once per CTA and shared by all its
// heads; a head only scales its x rows by b_j (in place) and its output rows
// by a_i.  With r1 the midpoint of the tile's prefix sums, the factors stay in
// [2^-60, 2^60] whenever the tile's decay spans at most 120 (log2 units): the
// fast path.  There the block left of the diagonal (t = 1) uses the same
// boundary, since cs_j >= r1 makes b_j <= dt_j for j < 128: G_10 (b * X_0)
// accumulates into Y, and the entering state term exp(cs_i) C_i h goes into a
// second accumulator ZW = C_t h^T scaled by alpha_i = exp(cs_i) <= 1.
// A head whose tile decays faster takes the exact path instead.  Its left
// block factorises through r = cs_{127} (both factors <= 1):
//   sum_{j < 128} G_ij exp(cs_i - cs_j) dt_j x_j
//      = alpha_i sum_j G_ij (beta_j x_j),   alpha_i = exp(cs_i - r), beta_j = exp(r - cs_j) dt_j,
// and with the entering state term alpha_i C_i (exp(r) h) it forms ZW =
// G_10 (beta x_{0..127}) + C_t (exp(r) h)^T (r = 0 for t = 0); its diagonal
// block is a per-element mask M_ij = G_ij exp(cs_i - cs_j) dt_j (j <= i) in TMEM, with each
// 32-column block below the diagonal factorised through the block's end (both
// factors <= 1) and exponentials per element only on the 32 x 32 diagonal
// blocks.  Output: y = a_i Y + alpha_i ZW + D_h x (a_i = 1 on the exact path);
// the x rows of the skip term reach the epilogue through TMEM: the warps that
// scale a head's x rows in shared memory first copy them, unscaled, to one of
// four TMEM slots.
//
// Roles (480 threads, 15 warps):
//   warps 0-7   prologue: G = C_t B^T (M = 128, N = 128 (t+1), K = dstate) is
//               copied from TMEM: the diagonal block becomes G o causal in bf16
//               (TMEM, the A operand of Y), the block to its left goes to
//               shared memory as bf16 (the A operand of G_10 X~); per head:
//               dt (held one token a thread, loaded a head ahead) and its prefix
//               sums, factors, then the x rows of the tile scaled by b_j (fast
//               path) or the exact mask written to TMEM (one slot), and for
//               t = 1 x rows 0..127 scaled by b_j (fast) or beta_j and h by
//               exp(r) (exact), in place; each warp reports its share of a
//               head's operands by its own mbarrier arrival;
//   warps 8-11  epilogue: y staged in shared memory, TMA store;
//   warp 12     TMA producer (x rows and entering states of the heads, a ring
//               of four slots for tile 0 of a 256-token chunk, two otherwise);
//   warp 13     MMA issuer and TMEM owner (G, Y, the left block, and on the
//               exact path ZW);
//   warp 14     with z2: second MMA issuer, ZW = C_t h^T on the fast path,
//               concurrently with warp 13's MMAs (a single thread issues an
//               MMA of these shapes no faster than one every few tens of ns,
//               whatever N, so two issuers halve a head's MMA time); a slot's
//               x/h and an accumulator are then released by both issuers'
//               commits.  Without z2 warp 13 issues ZW too and warp 14 idles
//               (where the scale warps bound the tile, the second stream of
//               MMA operand reads slows their shared-memory work more than it
//               saves).
// Every wait is bounded; a warpgroup leaves its loop only when all its
// threads agree (bar.red.or), so no named barrier is left half-arrived.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace ssd {
namespace outk {
using namespace sm100;

constexpr int kThreads = 480;
constexpr int kMaxHeads = 32;
constexpr float kLog2e = 1.4426950408889634f;

template <int Q, int N>
struct OutSmem {
    static constexpr int kNB = N / 64;                      // 64-wide blocks of dstate
    static constexpr int kHTile = kNB * 64 * 128;           // one head's h_prev (64 x N bf16)
    static constexpr int kC = 0;                            // C tile: kNB x 128 rows x 128 B
    static constexpr int kCBytes = kNB * 128 * 128;
    static constexpr int kBG = kC + kCBytes;                // B tile (prologue), then G_10 + h ring
    static constexpr int kG10Off = 0;                       // bf16 G_10, K-major SW128, 2 x 16 KB (t = 1)
    static constexpr int kHOff = (Q == 256) ? 32768 : 0;    // h ring of a t = 1 tile: 2 slots after G_10
    static constexpr int kBBytes = kNB * Q * 128;
    static constexpr int kBGBytes = (kBBytes > kHOff + 2 * kHTile) ? kBBytes : kHOff + 2 * kHTile;
    static constexpr int kXTile = Q * 128;                  // x rows [0, Q) of one head
    static constexpr int kX = kBG + kBGBytes;               // x ring: 2 slots of Q rows (or 4 of 128)
    static constexpr int kYs = kX + 2 * kXTile;             // y staging: 16 KB
    // per head modulo 4 (the scans of four heads are taken together)
    static constexpr int kDt = kYs + 128 * 128;             // float [4][Q] dt of a head
    static constexpr int kCs = kDt + 4 * Q * 4;             // float [4][Q] its prefix sums (log2 units)
    static constexpr int kWs = kCs + 4 * Q * 4;             // float [16]: per-warp sums of the scan
    static constexpr int kBeta = kWs + 16 * 4;              // float [4][128]  (t = 1 block left of diagonal)
    static constexpr int kBeta2 = kBeta + 4 * 128 * 4;      // float [4][128]  (diagonal block)
    static constexpr int kAl = kBeta2 + 4 * 128 * 4;        // float [4][128] alpha_i per factor slot
    static constexpr int kRow = kAl + 4 * 128 * 4;          // float [4][128] a_i (1: exact path)
    static constexpr int kPath = kRow + 4 * 128 * 4;        // int [4]: 1 = fast path
    static constexpr int kAD = kPath + 16;                  // float [2][kMaxHeads]: A_h (log2), D_h
    static constexpr int kBar = kAD + 2 * kMaxHeads * 4;    // mbarriers
    static constexpr int kTmem = kBar + 32 * 8;
    static constexpr int kFlags = kTmem + 16;
    static constexpr int kTotal = kFlags + 16;
    static constexpr int kAlloc = kTotal + 1024;
};

// mbarrier indices
enum {
    BAR_BC = 0, BAR_G = 1, BAR_GCONV = 2,
    BAR_XFULL = 3,      // up to four x/h ring slots
    BAR_XEMPTY = 7,
    BAR_MFULL = 11,     // four: the head's operands are ready (head modulo 4)
                        // 15: unused
    BAR_ACCFULL = 16, BAR_ACCEMPTY = 18,
    BAR_ALFULL = 20,    // four factor slots (alpha_i, a_i, path) per head modulo 4
    BAR_FEMPTY = 24,    // four: the epilogue has read the factor slot
    BAR_COUNT = 28
};

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColM = 0;       // bf16 exact-path mask, 64 columns (fp32 G_10 in the prologue)
constexpr uint32_t kColG = 128;     // fp32 diagonal block of G, 128 columns (prologue)
constexpr uint32_t kColGC = 128;    // then: bf16 G o causal, 64 columns
// unscaled bf16 x rows of the tile for the skip term, 4 slots of 32 columns
// (head modulo 4) in the columns the mask and G o causal leave free
__device__ __forceinline__ uint32_t col_xs(int f) { return f < 2 ? 64u + 32u * f : 192u + 32u * (f - 2); }
constexpr float kFastSpan = 120.f;  // largest tile decay (log2 units) of the fast path
constexpr uint32_t kColAcc = 256;   // two slots of 128: Y (64) then ZW (64)

// Scale the 16-byte pieces (8 bf16 each) of a shared-memory tile in place by a
// per-piece factor f(piece): 256 threads, NPER pieces each (piece t + 256 r for
// thread t); all loads are issued before any arithmetic.
template <int NPER, typename F>
__device__ __forceinline__ void scale_pieces(uint8_t* base, int t, F f) {
    uint4* p = reinterpret_cast<uint4*>(base);
    uint4 v[NPER];
    float sc[NPER];
#pragma unroll
    for (int r = 0; r < NPER; ++r) {
        v[r] = p[t + 256 * r];
        sc[r] = f(t + 256 * r);
    }
#pragma unroll
    for (int r = 0; r < NPER; ++r) {
        uint32_t* u = reinterpret_cast<uint32_t*>(&v[r]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u[e]));
            u[e] = pack_bf16x2(x.x * sc[r], x.y * sc[r]);
        }
        p[t + 256 * r] = v[r];
    }
}

// One tile: rows [128 t, 128 t + 128) of chunk c of sequence b, heads
// head0 .. head0 + HG - 1 (virtual heads of headdim 64; H counts them, real
// head = virtual head / ksplit).  `smem` is 1024-aligned.  When `progress`
// is given, the entering states are produced by walkers of the same launch,
// each of `whp` consecutive heads of one group (ceil(heads per group / whp)
// walkers a group, numbered by batch, group, first head): before loading the
// entering state of head h the producer waits until the count of h's walker
// has reached c + 1.
template <int Q, int N>
__device__ __forceinline__ void body(const CUtensorMap* tmX, const CUtensorMap* tmB,
                                     const CUtensorMap* tmC, const CUtensorMap* tmH,
                                     const CUtensorMap* tmY, const float* __restrict__ dt,
                                     const float* __restrict__ A, const float* __restrict__ Dv,
                                     int64_t L, int H, int G, int64_t T, int HG, int ksplit,
                                     int64_t b, int64_t c, int t, int head0, uint8_t* smem,
                                     const int* progress, int whp, bool z2,
                                     const WaitCtx& status) {
    // H counts virtual heads (headdim 64); real head = virtual head / ksplit
    const int Hr = H / ksplit;
    using S = OutSmem<Q, N>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t0 = c * Q;
    const int len = (int)((L - t0) < Q ? (L - t0) : Q);
    if (128 * t >= len) return;                 // tile entirely past the sequence end
    const int g = head0 / (H / G);
    const int KJ = 128 * (t + 1);               // columns j this tile needs
    const int row0 = 128 * t;                   // first row of the tile within the chunk
    // x/h ring: a tile-0 CTA of a 256-token chunk needs only 128 x rows and no
    // G_10, so its ring has four slots in the same space; otherwise two
    const int R = (Q == 256 && t == 0) ? 4 : 2;
    const int kXSlot = KJ * 128;                // bytes of one slot's x rows

    uint8_t* sC = smem + S::kC;
    uint8_t* sB = smem + S::kBG;
    uint8_t* sG10 = smem + S::kBG + S::kG10Off;
    uint8_t* sH = smem + S::kBG + (t == 1 ? S::kHOff : 0);
    uint8_t* sX = smem + S::kX;
    uint8_t* sY = smem + S::kYs;
    float* s_dt = reinterpret_cast<float*>(smem + S::kDt);
    float* s_cs = reinterpret_cast<float*>(smem + S::kCs);
    float* s_ws = reinterpret_cast<float*>(smem + S::kWs);
    float* s_beta = reinterpret_cast<float*>(smem + S::kBeta);
    float* s_beta2 = reinterpret_cast<float*>(smem + S::kBeta2);
    float* s_al = reinterpret_cast<float*>(smem + S::kAl);
    float* s_row = reinterpret_cast<float*>(smem + S::kRow);
    volatile int* s_path = reinterpret_cast<volatile int*>(smem + S::kPath);
    float* s_Ah = reinterpret_cast<float*>(smem + S::kAD);
    float* s_Dh = s_Ah + kMaxHeads;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + S::kFlags);   // [0]: any abort

    if (tid == 0) {
        // a head's operands are ready once each of the 8 scale warps has arrived;
        // a slot's x/h and an accumulator are released by both MMA issuers
        for (int i = 0; i < BAR_COUNT; ++i)
            mbar_init(&bars[i], (i >= BAR_MFULL && i < BAR_MFULL + 4) ? 8
                                : (z2 && ((i >= BAR_XEMPTY && i < BAR_XEMPTY + 4) ||
                                          (i >= BAR_ACCFULL && i < BAR_ACCFULL + 2))) ? 2 : 1);
        s_flag[0] = 0;
        fence_mbar_init();
    }
    if (warp == 13) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 12) {
        // ================================================== TMA producer
        if (lane == 0) {
            prefetch_tmap(tmX);
            prefetch_tmap(tmB);
            prefetch_tmap(tmC);
            prefetch_tmap(tmH);
            prefetch_tmap(tmY);
            mbar_expect_tx(&bars[BAR_BC], (uint32_t)(S::kCBytes + S::kNB * KJ * 128));
            for (int nb = 0; nb < S::kNB; ++nb) {
                tma_load_4d(sC + nb * 128 * 128, tmC, &bars[BAR_BC], nb * 64, g,
                            (int)(t0 + row0), (int)b);
                for (int rb = 0; rb <= t; ++rb)
                    tma_load_4d(sB + nb * Q * 128 + rb * 128 * 128, tmB, &bars[BAR_BC], nb * 64,
                                g, (int)(t0 + rb * 128), (int)b);
            }
            auto load_x = [&](int hi) {
                const int s = hi & (R - 1);
                mbar_expect_tx(&bars[BAR_XFULL + s], (uint32_t)(kXSlot + S::kHTile));
                for (int rb = 0; rb <= t; ++rb)
                    tma_load_4d(sX + s * kXSlot + rb * 128 * 128, tmX, &bars[BAR_XFULL + s], 0,
                                head0 + hi, (int)(t0 + rb * 128), (int)b);
            };
            auto load_h = [&](int hi) {
                const int s = hi & (R - 1);
                const int hrow = (int)(((b * T + c) * H + head0 + hi) * 64);
                for (int nb = 0; nb < S::kNB; ++nb)
                    tma_load_2d(sH + s * S::kHTile + nb * 64 * 128, tmH, &bars[BAR_XFULL + s],
                                nb * 64, hrow);
            };
            // entering states written by walkers of this launch: wait for the
            // walker of head hi to have written chunk c's
            int64_t ready_w = -1;
            auto wait_h = [&](int hi) -> bool {
                if (!progress) return true;
                const int h = head0 + hi, hpg = H / G, gg = h / hpg;
                const int wpg = (hpg + whp - 1) / whp;
                const int64_t w = (b * G + gg) * wpg + (h - gg * hpg) / whp;
                if (w <= ready_w) return true;
                ready_w = w;
                const bool r = flag_wait_geq(progress + w, (int)c + 1, status);
                fence_proxy_async_global();
                return r;
            };
            const int first = HG < R ? HG : R;
            for (int hi = 0; hi < first; ++hi) load_x(hi);
            // The h ring (and G_10) reuse the B tile's space: wait until G is
            // computed and copied out of TMEM.
            bool ok = mbar_wait(&bars[BAR_GCONV], 0, status);
            for (int hi = 0; hi < first && ok; ++hi) {
                ok = wait_h(hi);
                if (ok) load_h(hi);
            }
            for (int hi = R; hi < HG && ok; ++hi) {
                const int s = hi & (R - 1);
                ok = mbar_wait(&bars[BAR_XEMPTY + s], (uint32_t)((hi / R - 1) & 1), status);
                if (ok) load_x(hi);
                if (ok) ok = wait_h(hi);
                if (ok) load_h(hi);
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp == 13) {
        // ================================================== MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait(&bars[BAR_BC], 0, status);
            if (ok) {
                tc_fence_after();
                const uint32_t idesc_g = idesc_bf16_f32(128, KJ, false, false);
                const uint32_t c0 = smem_u32(sC), b0 = smem_u32(sB);
                const uint32_t dcol = (t == 1) ? 0u : kColG;   // t=1: [G_10 | G_11] over 256 columns
                for (int ks = 0; ks < N / 16; ++ks) {
                    const int nb = ks >> 2, ko = (ks & 3) * 32;
                    mma_ss(tmem + dcol, smem_desc_sw128(c0 + nb * 128 * 128 + ko, 16, 1024),
                           smem_desc_sw128(b0 + nb * Q * 128 + ko, 16, 1024), idesc_g, ks > 0);
                }
                mma_commit(&bars[BAR_G]);
            }
            const uint32_t idesc_y = idesc_bf16_f32(128, 64, false, true);    // A in TMEM, x MN-major
            const uint32_t idesc_w = idesc_bf16_f32(128, 64, false, true);    // G_10 K-major, x~ MN-major
            const uint32_t idesc_z = idesc_bf16_f32(128, 64, false, false);   // C, h both K-major
            const uint64_t gd = smem_desc_sw128(smem_u32(sG10), 16, 1024);
            const uint64_t cd = smem_desc_sw128(smem_u32(sC), 16, 1024);
            for (int hi = 0; hi < HG && ok; ++hi) {
                const int s = hi & (R - 1);           // x/h ring slot
                const int a = hi & 1;                 // accumulator slot
                const int f = hi & 3;                 // factor slot (path of the head)
                ok = mbar_wait(&bars[BAR_ALFULL + f], (uint32_t)((hi >> 2) & 1), status) &&
                     mbar_wait(&bars[BAR_XFULL + s], (uint32_t)((hi / R) & 1), status) &&
                     (hi < 2 || mbar_wait(&bars[BAR_ACCEMPTY + a], (uint32_t)(((hi >> 1) - 1) & 1),
                                          status));
                if (!ok) break;
                tc_fence_after();
                const uint32_t acc = tmem + kColAcc + 128 * a;
                // descriptors of each operand's first K step; a K step moves the start
                // address (16-byte units, low bits of the descriptor) by a constant
                const uint64_t xd = smem_desc_sw128(smem_u32(sX + s * kXSlot), 16, 1024);
                const uint64_t hd = smem_desc_sw128(smem_u32(sH + s * S::kHTile), 16, 1024);
                const bool fast = s_path[f] != 0;
                // ZW (+)= C_t h~^T.  On the fast path h is used as loaded, so these
                // MMAs go first (or to the second issuer), while the head's x rows are
                // still being scaled; on the exact path h exp(r) is ready only with
                // the rest.
                auto issue_z = [&](bool acc_first) {
#pragma unroll
                    for (int ks = 0; ks < N / 16; ++ks)
                        mma_ss(acc + 64, cd + (uint64_t)((ks >> 2) * 1024 + (ks & 3) * 2),
                               hd + (uint64_t)((ks >> 2) * 512 + (ks & 3) * 2), idesc_z, acc_first || ks > 0);
                };
                if (fast && !z2) issue_z(false);
                ok = mbar_wait(&bars[BAR_MFULL + f], (uint32_t)((hi >> 2) & 1), status);
                if (!ok) break;
                tc_fence_after();
                // Y = (G o causal) (b * X_t) [fast path] or M X_t [exact path] over the
                // diagonal block's 128 columns
                const uint32_t amat = fast ? tmem + kColGC : tmem + kColM;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts(acc, amat + ks * 8, xd + (uint64_t)((row0 / 16 + ks) * 128), idesc_y, ks > 0);
                // t = 1: G_10 times x rows 0..127, scaled by b_j like the diagonal
                // block's (fast path: into Y) or by beta_j (exact path: into ZW)
                const uint32_t wacc = fast ? acc : acc + 64;
                if (t == 1) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_ss(wacc, gd + (uint64_t)((ks >> 2) * 1024 + (ks & 3) * 2),
                               xd + (uint64_t)(ks * 128), idesc_w, fast || ks > 0);
                }
                if (!fast) issue_z(t == 1);
                mma_commit(&bars[BAR_XEMPTY + s]);           // x and h slot s: no reader left
                mma_commit(&bars[BAR_ACCFULL + a]);
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp == 14) {
        // ================================================== second MMA issuer (ZW, fast path)
        if (z2 && lane == 0) {
            const uint32_t idesc_z = idesc_bf16_f32(128, 64, false, false);   // C, h both K-major
            const uint64_t cd = smem_desc_sw128(smem_u32(sC), 16, 1024);
            bool ok = mbar_wait(&bars[BAR_BC], 0, status);                  // C has landed
            for (int hi = 0; hi < HG && ok; ++hi) {
                const int s = hi & (R - 1);
                const int a = hi & 1;
                const int f = hi & 3;
                ok = mbar_wait(&bars[BAR_ALFULL + f], (uint32_t)((hi >> 2) & 1), status) &&
                     mbar_wait(&bars[BAR_XFULL + s], (uint32_t)((hi / R) & 1), status) &&
                     (hi < 2 || mbar_wait(&bars[BAR_ACCEMPTY + a], (uint32_t)(((hi >> 1) - 1) & 1),
                                          status));
                if (!ok) break;
                tc_fence_after();
                if (s_path[f] != 0) {
                    const uint32_t acc = tmem + kColAcc + 128 * a;
                    const uint64_t hd = smem_desc_sw128(smem_u32(sH + s * S::kHTile), 16, 1024);
#pragma unroll
                    for (int ks = 0; ks < N / 16; ++ks)
                        mma_ss(acc + 64, cd + (uint64_t)((ks >> 2) * 1024 + (ks & 3) * 2),
                               hd + (uint64_t)((ks >> 2) * 512 + (ks & 3) * 2), idesc_z, ks > 0);
                }
                mma_commit(&bars[BAR_XEMPTY + s]);
                mma_commit(&bars[BAR_ACCFULL + a]);
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp < 8) {
        // ================================================== mask / scale warps (0-7)
        // Warp w owns TMEM lane quarter q = w % 4 (rows 32q..32q+31) and half
        // hf = w / 4 of the diagonal block's four 32-column blocks.
        const int q = warp & 3, hf = warp >> 2;
        const int m = q * 32 + lane;               // row within the tile
        const int i = row0 + m;                    // row within the chunk
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        // The prefix sums of dt*A are taken for four heads at a time: warp w
        // scans head slot k = w % 4 over half sg = w / 4 of the tile's KJ
        // columns, a lane holding kPer = KJ / 64 consecutive tokens, whose dt
        // it loads one batch of four heads ahead (the first while the
        // prologue runs).
        constexpr int kPerMax = Q / 64;
        const int per = KJ / 64;
        const int sk = warp & 3, sg = warp >> 2;
        const int jseg = sg * (KJ / 2) + lane * per;          // this lane's first token
        float dnext[kPerMax];
        auto load_dt = [&](int hb) {                          // heads hb .. hb + 3
#pragma unroll
            for (int e = 0; e < kPerMax; ++e) {
                const int j = jseg + e;
                dnext[e] = (e < per && j < len && hb + sk < HG)
                               ? dt[(b * L + t0 + j) * Hr + (head0 + hb + sk) / ksplit] : 0.f;
            }
        };
        load_dt(0);
        if (tid < HG) {
            s_Ah[tid] = A[(head0 + tid) / ksplit] * kLog2e;
            s_Dh[tid] = Dv[(head0 + tid) / ksplit];
        }
        named_bar_sync(1, 256);
        bool fail = !mbar_wait(&bars[BAR_G], 0, status);
        if (!named_bar_or(1, 256, fail)) {
            tc_fence_after();
            if (t == 1) {
                // G_10 (TMEM columns [0, 128)) -> bf16 K-major SW128 tile: K-block
                // kb = j / 64, row m at 128 B, 16-byte chunk c at (c ^ (m & 7)).
                for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + cb * 32, r);
                    uint4* row = reinterpret_cast<uint4*>(sG10 + (cb >> 1) * 16384 + m * 128);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int lc = (cb & 1) * 4 + u;
                        row[lc ^ (m & 7)] = make_uint4(
                            pack_bf16x2(__uint_as_float(r[8 * u + 0]), __uint_as_float(r[8 * u + 1])),
                            pack_bf16x2(__uint_as_float(r[8 * u + 2]), __uint_as_float(r[8 * u + 3])),
                            pack_bf16x2(__uint_as_float(r[8 * u + 4]), __uint_as_float(r[8 * u + 5])),
                            pack_bf16x2(__uint_as_float(r[8 * u + 6]), __uint_as_float(r[8 * u + 7])));
                    }
                }
                fence_proxy_async_smem();          // G_10 is read by the MMA (async proxy)
            }
            // Blocks above the diagonal (column block cb > quarter q) are zero in
            // every head's mask: write them once -- after every warp has finished
            // reading G_10 out of the same TMEM columns.
            tc_fence_before();
            named_bar_sync(1, 256);
            tc_fence_after();
            {
                uint32_t zeros[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) zeros[u] = 0u;
                for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb)
                    if (cb > q) tmem_st16(tmem + lane_base + kColM + 16 * cb, zeros);
            }
            {
                // G o causal -> bf16 at kColGC, over the fp32 columns it is made
                // from: every warp reads its two 32-column blocks, then all write.
                uint32_t pk[2][16];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int cb = 2 * hf + h2;
                    uint32_t gr[32];
                    tmem_ld32(tmem + lane_base + kColG + 32 * cb, gr);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int jj = 32 * cb + 2 * e;  // column within the tile
                        pk[h2][e] = pack_bf16x2(jj <= m ? __uint_as_float(gr[2 * e]) : 0.f,
                                                jj + 1 <= m ? __uint_as_float(gr[2 * e + 1]) : 0.f);
                    }
                }
                tc_fence_before();
                named_bar_sync(1, 256);
                tc_fence_after();
                tmem_st16(tmem + lane_base + kColGC + 16 * (2 * hf), pk[0]);
                tmem_st16(tmem + lane_base + kColGC + 16 * (2 * hf + 1), pk[1]);
            }
            tc_fence_before();
            named_bar_sync(1, 256);
            if (tid == 0) mbar_arrive(&bars[BAR_GCONV]);

            for (int hi = 0; hi < HG; ++hi) {
                const int s = hi & (R - 1);           // x/h ring slot
                const int f = hi & 3;                 // factor slot and skip-term x slot
                if ((hi & 3) == 0) {
                    // inclusive prefix sums of dt*A (log2 units) of heads hi .. hi + 3
                    // over the tile's KJ columns: a shuffle scan per warp segment,
                    // then the first segment's total as the second's offset.  The
                    // slots written are those of heads hi - 4 .. hi - 1, which every
                    // thread has finished with once it reaches the first barrier.
                    float dcur[kPerMax], v[kPerMax];
#pragma unroll
                    for (int e = 0; e < kPerMax; ++e) dcur[e] = dnext[e];
                    if (hi + 4 < HG) load_dt(hi + 4);
                    const float Ak = hi + sk < HG ? s_Ah[hi + sk] : 0.f;
                    float run = 0.f;
#pragma unroll
                    for (int e = 0; e < kPerMax; ++e) {
                        run += dcur[e] * Ak;              // tokens past KJ or L add 0
                        v[e] = run;
                    }
                    float incl = run;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float u = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += u;
                    }
                    if (lane == 31) s_ws[warp] = incl;
                    named_bar_sync(1, 256);
                    const float off = (incl - run) + (sg ? s_ws[sk] : 0.f);
                    float* csk = s_cs + sk * Q;
                    float* dtk = s_dt + sk * Q;
#pragma unroll
                    for (int e = 0; e < kPerMax; ++e)
                        if (e < per) {
                            csk[jseg + e] = v[e] + off;
                            dtk[jseg + e] = dcur[e];
                        }
                    named_bar_sync(1, 256);
                }
                // factor slot f is free once the epilogue of head hi - 4 has read it
                // (each thread waits before writing it; the barrier that publishes
                // the factors below also shares the outcome)
                fail = hi >= 4 && !mbar_wait(&bars[BAR_FEMPTY + f], (uint32_t)(((hi >> 2) - 1) & 1), status);
                const float* cs = s_cs + f * Q;
                const float* hdt = s_dt + f * Q;
                float* beta = s_beta + f * 128;
                float* beta2 = s_beta2 + f * 128;
                const float cs_i = cs[i];
                const float r = (t == 1) ? cs[127] : 0.f;
                // the tile's decay span decides the path (the same for every thread)
                const float c_first = cs[row0], c_last = cs[row0 + 127];
                const float r1 = 0.5f * (c_first + c_last);
                // fast path: the tile's own factors stay within 2^+-60; for t = 1 the
                // left block's b_j = 2^(r1 - cs_j) dt_j must too, which holds for any
                // A <= 0 (cs_j >= r1) and bounds a growing state (A > 0)
                const bool fast = fabsf(c_last - c_first) <= kFastSpan &&
                                  (t == 0 || r1 - cs[0] <= 0.5f * kFastSpan);
                if (hf == 0) {
                    if (t == 1) beta[m] = fast_exp2((fast ? r1 : r) - cs[m]) * hdt[m];
                    s_al[f * 128 + m] = fast_exp2(fast ? cs_i : cs_i - r);
                    s_row[f * 128 + m] = fast ? fast_exp2(cs_i - r1) : 1.f;
                } else {
                    // fast: b_j; exact: beta of j through the end of its 32-column block
                    const int j = row0 + m;
                    beta2[m] = fast_exp2((fast ? r1 : cs[row0 + (m | 31)]) - cs[j]) * hdt[j];
                }
                if (tid == 0) s_path[f] = fast ? 1 : 0;
                // the exact path writes the mask slot: free once the MMAs of head hi - 1
                // have completed, which the end of that head's epilogue implies (a wait
                // on the MMAs' own commit could alias: the scale warps may be more than
                // one head ahead of the MMAs, while the epilogue of head hi - 5 is
                // known to be done, so this barrier lags by at most one phase); both
                // paths need the head's x rows and entering state
                fail = fail ||
                       (!fast && hi >= 1 &&
                        !mbar_wait(&bars[BAR_FEMPTY + ((hi - 1) & 3)],
                                   (uint32_t)(((hi - 1) >> 2) & 1), status)) ||
                       !mbar_wait(&bars[BAR_XFULL + s], (uint32_t)((hi / R) & 1), status);
                if (named_bar_or(1, 256, fail)) break;   // also publishes the factors
                if (tid == 0) mbar_arrive(&bars[BAR_ALFULL + f]);
                if (t == 1) {
                    // x rows 0..127 *= b_j (fast path) or beta_j (exact path), row j =
                    // piece / 8; on the exact path also h *= exp(r); in place
                    scale_pieces<4>(sX + s * kXSlot, tid, [&](int k) { return beta[k >> 3]; });
                    if (!fast) {
                        const float er = fast_exp2(r);
                        scale_pieces<S::kHTile / 4096>(sH + s * S::kHTile, tid, [&](int) { return er; });
                    }
                }
                {
                    // The tile's x rows: warp (q, hf) takes row m, 16-byte chunks
                    // 4 hf .. 4 hf + 3 (stored at chunk ^ (m & 7)).  Unscaled, they go to
                    // TMEM slot f (columns = element / 2) for the epilogue's skip term;
                    // on the fast path they are then scaled by b_m in place (the MMA's
                    // B operand).
                    uint4* xrow = reinterpret_cast<uint4*>(sX + s * kXSlot + (row0 + m) * 128);
                    uint4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) v[u] = xrow[(4 * hf + u) ^ (m & 7)];
                    {
                        uint32_t w[16];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            w[4 * u + 0] = v[u].x; w[4 * u + 1] = v[u].y;
                            w[4 * u + 2] = v[u].z; w[4 * u + 3] = v[u].w;
                        }
                        tc_fence_after();          // slot f's previous reader (head hi - 4) is done
                        tmem_st16(tmem + lane_base + col_xs(f) + 16 * hf, w);
                    }
                    if (fast) {
                        const float bm = beta2[m];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            uint32_t* e4 = reinterpret_cast<uint32_t*>(&v[u]);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 xf = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&e4[e]));
                                e4[e] = pack_bf16x2(xf.x * bm, xf.y * bm);
                            }
                            xrow[(4 * hf + u) ^ (m & 7)] = v[u];
                        }
                    }
                }
                fence_proxy_async_smem();
                tc_fence_after();

                // exact path: diagonal-block mask -> the TMEM mask slot (64 columns of
                // bf16 pairs), from the bf16 G o causal
                for (int cb = 2 * hf; cb < 2 * hf + 2 && !fast; ++cb) {
                    const int j0 = row0 + 32 * cb;
                    uint32_t packed[16];
                    if (cb > q) continue;                 // zero block, written once
                    {
                        uint32_t gr[32];
                        {
                            uint32_t gp[16];
                            tmem_ld16(tmem + lane_base + kColGC + 16 * cb, gp);
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                gr[2 * e] = gp[e] << 16;
                                gr[2 * e + 1] = gp[e] & 0xffff0000u;
                            }
                        }
                        if (cb < q) {
                            // entirely below the diagonal: factorised through the block's end
                            const float alpha = fast_exp2(cs_i - cs[j0 + 31]);
                            const float4* bet = reinterpret_cast<const float4*>(beta2 + 32 * cb);
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const float4 bv = bet[u];
                                packed[2 * u] = pack_bf16x2(__uint_as_float(gr[4 * u]) * alpha * bv.x,
                                                            __uint_as_float(gr[4 * u + 1]) * alpha * bv.y);
                                packed[2 * u + 1] =
                                    pack_bf16x2(__uint_as_float(gr[4 * u + 2]) * alpha * bv.z,
                                                __uint_as_float(gr[4 * u + 3]) * alpha * bv.w);
                            }
                        } else {
                            // 32 x 32 block on the diagonal: exact exponentials, causal mask
#pragma unroll
                            for (int u = 0; u < 16; ++u) {
                                const int ja = j0 + 2 * u, jb = ja + 1;
                                const float va = (ja <= i)
                                    ? __uint_as_float(gr[2 * u]) * fast_exp2(cs_i - cs[ja]) * hdt[ja] : 0.f;
                                const float vb = (jb <= i)
                                    ? __uint_as_float(gr[2 * u + 1]) * fast_exp2(cs_i - cs[jb]) * hdt[jb] : 0.f;
                                packed[u] = pack_bf16x2(va, vb);
                            }
                        }
                    }
                    tmem_st16(tmem + lane_base + kColM + 16 * cb, packed);
                }
                // Each warp reports its share (scaled rows, mask blocks) by itself.  No
                // block barrier is needed here: the factors, sums and dt of a head
                // live in slot hi % 4, which is rewritten only after the next batch
                // scan's first barrier, and the shared mask slot (exact path) only
                // after the next head's factor barrier.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[BAR_MFULL + f]);
            }
        }
        if (fail) s_flag[0] = 1;
    } else {
        // ================================================== epilogue warpgroup (warps 8-11)
        // y rows go to a 128-byte-swizzled staging tile and leave by TMA store
        // (coalesced; rows past the sequence end are clipped by the tensor map).
        const int m = tid - 256;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        bool fail = false;
        for (int hi = 0; hi < HG; ++hi) {
            const int s = hi & 1;
            fail = !(mbar_wait(&bars[BAR_ACCFULL + s], (uint32_t)((hi >> 1) & 1), status) &&
                     mbar_wait(&bars[BAR_ALFULL + (hi & 3)], (uint32_t)((hi >> 2) & 1), status));
            // the staging tile is free once the previous head's store has read it
            if (m == 0) bulk_wait_group_read<0>();
            if (named_bar_or(2, 128, fail)) break;
            tc_fence_after();
            const float al = s_al[(hi & 3) * 128 + m];
            const float ar = s_row[(hi & 3) * 128 + m];
            const float Dh = s_Dh[hi];
            uint4* ystage = reinterpret_cast<uint4*>(sY + m * 128);
            const uint32_t acc = tmem + lane_base + kColAcc + 128 * s;
            const uint32_t xs = tmem + lane_base + col_xs(hi & 3);   // unscaled x row
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                // columns 16 qq .. 16 qq + 15 of Y and ZW, x elements 16 qq .. 16 qq + 15
                uint32_t yr[16], zr[16], xw[8];
                tmem_ld16x2_8(acc + 16 * qq, acc + 64 + 16 * qq, xs + 8 * qq, yr, zr, xw);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int lc = 2 * qq + u;     // logical 16-byte chunk of the row
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 xf =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[4 * u + e]));
                        const int k = 8 * u + 2 * e;
                        const float v0 =
                            fmaf(al, __uint_as_float(zr[k]), ar * __uint_as_float(yr[k])) + Dh * xf.x;
                        const float v1 =
                            fmaf(al, __uint_as_float(zr[k + 1]), ar * __uint_as_float(yr[k + 1])) + Dh * xf.y;
                        o[e] = pack_bf16x2(v0, v1);
                    }
                    ystage[lc ^ (m & 7)] = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(2, 128);
            if (m == 0) {
                tma_store_4d(tmY, sY, 0, head0 + hi, (int)(t0 + row0), (int)b);
                bulk_commit_group();
                mbar_arrive(&bars[BAR_ACCEMPTY + s]);
                mbar_arrive(&bars[BAR_FEMPTY + (hi & 3)]);
            }
        }
        if (m == 0) bulk_wait_group<0>();      // stores done before the CTA leaves
        if (fail) s_flag[0] = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (s_flag[0] && tid == 12 * 32) {
        // A wait gave up somewhere: before the CTA's shared memory and TMEM
        // go away, give outstanding TMA loads and MMAs a last (bounded) chance
        // to land.  Waiting on already-completed phases returns at once.
        for (int k = 0; k < R && k < HG; ++k) mbar_wait(&bars[BAR_XFULL + k], 0, status);
        for (int k = 0; k < 2 && k < HG; ++k) mbar_wait(&bars[BAR_ACCFULL + k], 0, status);
        mbar_wait(&bars[BAR_BC], 0, status);
        mbar_wait(&bars[BAR_G], 0, status);
    }
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Heads per tile: the largest divisor of the heads per group up to kMaxHeads.
inline int pick_heads_per_cta(int64_t H, int64_t G) {
    const int64_t hpg = H / G;
    for (int hg = kMaxHeads; hg > 1; --hg)
        if (hpg % hg == 0) return hg;
    return 1;
}

}  // namespace outk
}  // namespace ssd
