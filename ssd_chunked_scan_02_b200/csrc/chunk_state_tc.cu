// chunk_state_tc.cu -- chunk states on the tcgen05 tensor cores (bf16 inputs,
// fp32 accumulation), steps a0 + a2 of the block-decomposed SSD forward:
//
//   cs_j  = sum_{k <= j} dt_k A_h           (inclusive prefix, fp32, warp shuffles)
//   w_j   = exp(cs_last - cs_j) dt_j        (decay to the chunk's end, times dt)
//   S[p, n] = sum_j (w_j x_j[p]) B_j[n]    (P x N chunk state, zero start)
//
// The backward's reverse pass uses the same contraction with w_j = exp(cs_j)
// (the decay from the chunk's start), dy in x's place and C in B's:
// sum_j exp(cs_j) dy_j C_j^T is what a chunk adds to dL/dh of the state
// entering it.
//
// "Transformers are SSMs" (CiteArk), AI research summary: the state a chunk
// hands on is one dense contraction over the chunk's tokens (B^T (w * X)),
// which is what the tensor cores are for.
//
// Persistent kernel: one CTA per SM walks a contiguous range of work items,
// an item being one head pair of one (batch, chunk); items are ordered
// (batch, chunk, pair), so a CTA reloads the chunk's B tile only where its
// range crosses into another chunk (or B/C group).  With dstate N = 128 an
// item computes S^T (M = N state rows, N = two heads x P = 64 columns): A =
// the chunk's B tile, B = the pair's scaled x tiles, so a TMEM lane is a state
// column n.  With N = 64 it computes S (M = two heads x P rows, N = dstate).
// Both operands are MN-major 128-byte-swizzled tiles brought by TMA; x comes
// through a six-stage ring of 64-token pair tiles (16 KB), so loads of the
// next items stream while the current one is scaled, multiplied and stored.
// Roles:
//   warp 12 (one lane)  TMA producer: B tile per chunk, x stages into the ring;
//   warps 0-7           dt prefix sums and w_j per item (each warp loads its
//                       own 64-token segment of one head's dt, the next item's
//                       while the current one is scaled), then x rows scaled
//                       in place by w_j (the MMA sees bf16(w_j x_j)); each warp
//                       reports a stage scaled by its own mbarrier arrival;
//   warp 13 (one lane)  MMA issuer (and TMEM owner), two accumulator slots;
//   warps 8-11          epilogue: TMEM -> fp32 S in HBM, layout (b, T, H, P, N),
//                       through a shared-memory staging pair and TMA bulk
//                       stores (N = 128: 32 x 128 fp32 boxes; N = 64: 128 x 32,
//                       128-byte swizzled).
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
constexpr int kRing = 6;          // x ring stages
constexpr int kStageTok = 64;     // tokens per ring stage

template <int Q, int N>
struct StateSmem {
    static constexpr int kStages = Q / kStageTok;          // ring stages per item
    static constexpr int kHeadStage = kStageTok * 128;     // one head: 64 tokens x 64 bf16 (8 KB)
    static constexpr int kStage = 2 * kHeadStage;          // one ring stage: a head pair (16 KB)
    static constexpr int kB = 0;                           // N/64 blocks of Q rows x 128 B
    static constexpr int kBBytes = (N / 64) * Q * 128;
    static constexpr int kX = kB + kBBytes;
    static constexpr int kOut = kX + kRing * kStage;       // N = 128: 2 x [32][128] fp32 staging
    static constexpr int kOutBytes = 2 * 32 * 128 * 4;     // two 16 KB staging boxes
    static constexpr int kW = kOut + kOutBytes;            // float [2 buffers][2 heads][Q]: w_j
    static constexpr int kSeg = kW + 4 * Q * 4;            // float [8]: prefix segment sums
    static constexpr int kBar = kSeg + 8 * 4;
    static constexpr int kTmem = kBar + 32 * 8;
    static constexpr int kCnt = kTmem + 16;                // producer's issue counts
    static constexpr int kFlags = kCnt + 16;
    static constexpr int kTotal = kFlags + 16;
    static constexpr int kAlloc = kTotal + 1024;           // slack to align the base to 1 KB
    static constexpr uint32_t kTmemCols = (2 * N <= 128) ? 128 : 256;   // two fp32 D slots
};

enum {
    BAR_B = 0,
    BAR_XFULL = 1,
    BAR_XSCALED = BAR_XFULL + kRing,
    BAR_XEMPTY = BAR_XSCALED + kRing,
    BAR_ACCFULL = BAR_XEMPTY + kRing,
    BAR_ACCEMPTY = BAR_ACCFULL + 2,
    BAR_DRAIN = BAR_ACCEMPTY + 2,
    BAR_COUNT = BAR_DRAIN + 1
};
static_assert(BAR_COUNT <= 32, "barrier area");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Walks work items in order: i -> (batch, chunk, head pair), advanced by
// counters (one division per CTA, at the start); key names the B tile used.
// Pairs are pairs of (virtual) heads of one group (HeadPairs).
struct ItemIter {
    int64_t b, c, T;
    int pair, pairs, ppg, G;
    __device__ __forceinline__ void init(int64_t i, int pairs_, int64_t T_, int ppg_, int G_) {
        pairs = pairs_;
        T = T_;
        ppg = ppg_;
        G = G_;
        const int64_t bc = i / pairs;
        pair = (int)(i - bc * pairs);
        c = bc % T;
        b = bc / T;
    }
    __device__ __forceinline__ void next() {
        if (++pair < pairs) return;
        pair = 0;
        if (++c < T) return;
        c = 0;
        ++b;
    }
    __device__ __forceinline__ int g() const { return pair / ppg; }
    __device__ __forceinline__ int64_t key() const { return (b * T + c) * G + g(); }
};

template <int Q, int N>
__global__ void __launch_bounds__(kThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmS,
                      const __grid_constant__ CUtensorMap tmS1, const float* __restrict__ dt,
                      const float* __restrict__ A, float* __restrict__ states,
                      float* __restrict__ logdecay, int64_t L, int H, int G, int64_t T,
                      int64_t items, int ksplit, int rev, WaitCtx status) {
    using S = StateSmem<Q, N>;
    constexpr bool kTrans = (N == 128);
    constexpr int kSt = S::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sB = smem + S::kB;
    uint8_t* sX = smem + S::kX;
    float* s_out = reinterpret_cast<float*>(smem + S::kOut);
    float* s_w = reinterpret_cast<float*>(smem + S::kW);
    float* s_seg = reinterpret_cast<float*>(smem + S::kSeg);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile uint32_t* s_cnt = reinterpret_cast<volatile uint32_t*>(smem + S::kCnt);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + S::kFlags);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // H counts virtual heads (headdim 64); real head = virtual head / ksplit
    const HeadPairs hp(H, G);
    const int pairs = G * hp.per_group(), ppg = hp.per_group();
    const int Hr = H / ksplit;
    const int64_t i0 = (int64_t)blockIdx.x * items / gridDim.x;
    const int64_t i1 = (int64_t)(blockIdx.x + 1) * items / gridDim.x;

    if (tid == 0) {
        // a stage counts as scaled once each of the 8 scale warps has arrived
        for (int i = 0; i < BAR_COUNT; ++i)
            mbar_init(&bars[i], (i >= BAR_XSCALED && i < BAR_XSCALED + kRing) ? 8 : 1);
        s_flag[0] = 0;
        s_cnt[0] = 0;
        s_cnt[1] = 0;
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
            bool ok = true;
            uint32_t it = 0, nb = 0;
            int64_t key_prev = -1;
            ItemIter w;
            w.init(i0, pairs, T, ppg, G);
            for (int64_t i = i0; i < i1 && ok; ++i, w.next()) {
                const int t0 = (int)(w.c * Q);
                const int64_t key = w.key();
                if (key != key_prev) {
                    // The B buffer is single: before replacing it, every MMA that
                    // reads it (up to the last stage issued) must have completed.
                    if (it > 0)
                        ok = mbar_wait(&bars[BAR_XEMPTY + (it - 1) % kRing],
                                       ((it - 1) / kRing) & 1, status);
                    if (!ok) break;
                    mbar_expect_tx(&bars[BAR_B], S::kBBytes);
                    for (int q = 0; q < N / 64; ++q)
                        tma_load_4d(sB + q * Q * 128, &tmB, &bars[BAR_B], q * 64, w.g(), t0,
                                    (int)w.b);
                    ++nb;
                    key_prev = key;
                }
                int gg, h0;
                bool has1;
                hp.map(w.pair, &gg, &h0, &has1);
                const int h1x = has1 ? h0 + 1 : H;    // the phantom's x: out of range, zeros
                for (int st = 0; st < kSt; ++st) {
                    const uint32_t slot = it % kRing;
                    if (it >= kRing)
                        ok = mbar_wait(&bars[BAR_XEMPTY + slot], ((it / kRing) - 1) & 1, status);
                    if (!ok) break;
                    uint8_t* dst = sX + slot * S::kStage;
                    mbar_expect_tx(&bars[BAR_XFULL + slot], S::kStage);
                    tma_load_4d(dst, &tmX, &bars[BAR_XFULL + slot], 0, h0, t0 + st * kStageTok,
                                (int)w.b);
                    tma_load_4d(dst + S::kHeadStage, &tmX, &bars[BAR_XFULL + slot], 0, h1x,
                                t0 + st * kStageTok, (int)w.b);
                    ++it;
                }
            }
            s_cnt[0] = it;
            s_cnt[1] = nb;
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp == 13) {
        // ================================================== MMA issuer
        if (lane == 0) {
            // N = 128: D = S^T = B^T (w x) (M = 128 state rows, N = 128 pair columns);
            // N = 64:  D = S   = (w x)^T B (M = 128 pair rows, N = 64 state columns).
            constexpr uint32_t kIdesc = idesc_bf16_f32(128, kTrans ? 128 : N, true, true);
            constexpr uint32_t kSlotCols = kTrans ? 128 : N;
            const uint32_t b0 = smem_u32(sB), x0 = smem_u32(sX);
            bool ok = true;
            uint32_t it = 0, nb = 0, k = 0;
            int64_t key_prev = -1;
            ItemIter w;
            w.init(i0, pairs, T, ppg, G);
            for (int64_t i = i0; i < i1 && ok; ++i, ++k, w.next()) {
                const int64_t key = w.key();
                if (key != key_prev) {
                    ok = mbar_wait(&bars[BAR_B], nb & 1, status);
                    if (!ok) break;
                    ++nb;
                    key_prev = key;
                }
                const uint32_t as = k & 1;
                if (k >= 2) ok = mbar_wait(&bars[BAR_ACCEMPTY + as], ((k >> 1) - 1) & 1, status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d = tmem + as * kSlotCols;
                for (int st = 0; st < kSt; ++st, ++it) {
                    const uint32_t slot = it % kRing;
                    ok = mbar_wait(&bars[BAR_XSCALED + slot], (it / kRing) & 1, status);
                    if (!ok) break;
                    tc_fence_after();
                    for (int ks = 0; ks < kStageTok / 16; ++ks) {
                        // x pair: two 64-column atoms (heads) kHeadStage apart; B: 64-column
                        // atoms of dstate Q * 128 apart; 8-row groups 1024 B apart.
                        const uint64_t xd =
                            smem_desc_sw128(x0 + slot * S::kStage + ks * 2048, S::kHeadStage, 1024);
                        const uint64_t bd = smem_desc_sw128(
                            b0 + (uint32_t)(st * kStageTok + ks * 16) * 128, Q * 128, 1024);
                        if (kTrans) mma_ss(d, bd, xd, kIdesc, (st | ks) != 0);
                        else mma_ss(d, xd, bd, kIdesc, (st | ks) != 0);
                    }
                    mma_commit(&bars[BAR_XEMPTY + slot]);
                }
                if (!ok) break;
                mma_commit(&bars[BAR_ACCFULL + as]);
            }
            mma_commit(&bars[BAR_DRAIN]);
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp < 8) {
        // ================================================== dt / scale warps (0-7)
        // Per item: (a0) the pair's dt for the chunk, loaded by warp (head hk =
        // w / 4, segment sg = w % 4) straight for its Q / 4 tokens (the next
        // item's dt is loaded while the current one is scaled); the inclusive
        // prefix sum of dt*A per segment (Q / 128 consecutive tokens a lane, a
        // shuffle scan of the lane totals), segment offsets through shared
        // memory, and w_j = exp(cs_last - cs_j) dt_j; then each x row j scaled
        // by w_j.
        constexpr int kPer = Q / 128;         // tokens per lane of a segment
        constexpr int kSegTok = Q / 4;        // tokens per segment
        const int hk = warp >> 2, sg = warp & 3;
        float dreg[kPer];
        auto head_of = [&](const ItemIter& w, bool* real) {
            int gg, h0;
            bool has1;
            hp.map(w.pair, &gg, &h0, &has1);
            *real = hk == 0 || has1;
            return h0 + hk;
        };
        auto load_dt = [&](const ItemIter& w) {
            const int64_t t0 = w.c * Q;
            const int64_t len = (L - t0) < Q ? (L - t0) : Q;
            bool real;
            const int hv = head_of(w, &real);
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int j = sg * kSegTok + lane * kPer + k;
                dreg[k] = (real && j < len) ? dt[(w.b * L + t0 + j) * Hr + hv / ksplit] : 0.f;
            }
        };
        // w_j of the item into buffer buf (published by the caller's barrier)
        auto prefix = [&](const ItemIter& w, int buf) {
            bool real;
            const int hv = head_of(w, &real);
            const float Ah = real ? A[hv / ksplit] : 0.f;
            float v[kPer];
            float run = 0.f;                       // tokens past the sequence end add 0
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                run += dreg[k] * Ah;
                v[k] = run;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            if (lane == 31) s_seg[warp] = incl;
            named_bar_sync(1, 256);
            float off = incl - run, last = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float sq = s_seg[hk * 4 + q];
                if (q < sg) off += sq;
                last += sq;
            }
            float* wk = s_w + (buf * 2 + hk) * Q + sg * kSegTok + lane * kPer;
#pragma unroll
            for (int k = 0; k < kPer; ++k)
                wk[k] = rev ? expf(v[k] + off) : expf(last - (v[k] + off)) * dreg[k];
            // one log-decay per real head: the first of its virtual heads writes it
            if (sg == 0 && lane == 0 && real && hv % ksplit == 0)
                logdecay[(w.b * T + w.c) * Hr + hv / ksplit] = last;
        };

        bool fail = false;
        uint32_t it = 0;
        ItemIter wn;
        wn.init(i0, pairs, T, ppg, G);
        if (i0 < i1) {
            load_dt(wn);
            prefix(wn, 0);
        }
        named_bar_sync(1, 256);
        for (int64_t i = i0, k = 0; i < i1 && !fail; ++i, ++k) {
            const bool has_next = i + 1 < i1;
            wn.next();                          // item i + 1
            if (has_next) load_dt(wn);
            const float* wbuf = s_w + (k & 1) * 2 * Q;
            // Each warp scales its own rows of a stage and reports it scaled by
            // itself (a stage's barrier counts 8 arrivals): no block barrier per
            // stage.  A failed wait makes the warp stop arriving; the verdict is
            // shared once per item, after the next item's prefix sums.
            for (int st = 0; st < kSt && !fail; ++st, ++it) {
                const uint32_t slot = it % kRing;
                if (!mbar_wait(&bars[BAR_XFULL + slot], (it / kRing) & 1, status)) {
                    fail = true;
                    break;
                }
                // (a2 operand) 128 rows (two heads x 64 tokens) of 8 16-byte chunks;
                // a warp covers four whole rows per access (no bank conflicts).
                uint4* tile = reinterpret_cast<uint4*>(sX + slot * S::kStage);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int idx = tid + 256 * q, row = idx >> 3;
                    const float wj = wbuf[(row >> 6) * Q + st * kStageTok + (row & 63)];
                    uint4 v = tile[idx];
                    uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u[e]));
                        u[e] = pack_bf16x2(f.x * wj, f.y * wj);
                    }
                    tile[idx] = v;
                }
                fence_proxy_async_smem();       // generic writes -> visible to the MMA (async proxy)
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[BAR_XSCALED + slot]);
            }
            if (has_next) prefix(wn, (int)((k + 1) & 1));
            // publishes the next item's w_j and shares the verdict of the waits
            if (named_bar_or(1, 256, fail)) {
                fail = true;
                break;
            }
        }
        if (fail) s_flag[0] = 1;
    } else {
        // ================================================== epilogue warps (8-11)
        const int m = tid - 256;                 // TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        bool fail = false;
        uint32_t q = 0;                          // staging boxes written so far
        int64_t k = 0;
        ItemIter w;
        w.init(i0, pairs, T, ppg, G);
        for (int64_t i = i0; i < i1; ++i, ++k, w.next()) {
            const uint32_t as = (uint32_t)(k & 1);
            const bool miss = !mbar_wait(&bars[BAR_ACCFULL + as], (uint32_t)((k >> 1) & 1), status);
            if (named_bar_or(2, 128, miss)) {
                fail = true;
                break;
            }
            tc_fence_after();
            if (kTrans) {
                // lane m = state column n; column c = (head c / 64, p = c % 64).  The
                // pair's 128 (head, p) rows of S are contiguous in HBM; each 32-column
                // block goes out as one 32 x 128 fp32 box.
                int gg, h0;
                bool has1;
                hp.map(w.pair, &gg, &h0, &has1);
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc, ++q) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + as * 128 + cc * 32, r);
                    float* buf = s_out + (q & 1) * (32 * 128);
                    if (m == 0) bulk_wait_group_read<1>();   // the store of two boxes ago is read
                    named_bar_sync(2, 128);
#pragma unroll
                    for (int e = 0; e < 32; ++e) buf[e * 128 + m] = __uint_as_float(r[e]);
                    fence_proxy_async_smem();
                    if (cc == 3) tc_fence_before();
                    named_bar_sync(2, 128);
                    if (m == 0) {
                        if (cc == 3) mbar_arrive(&bars[BAR_ACCEMPTY + as]);
                        // (the phantom's rows, cc >= 2 without a second head, are not stored)
                        if (cc < 2 || has1)
                            tma_store_3d(&tmS, buf, 0, h0 * 64 + cc * 32, (int)(w.b * T + w.c));
                        bulk_commit_group();
                    }
                }
            } else {
                // lane m = (head m / 64, p = m % 64); columns = state n.  Each 32-column
                // block of the pair's 128 rows goes out as one 128 x 32 fp32 box (64 x
                // 32 for a head paired with a phantom), staged with the 128-byte
                // swizzle (chunk c of row m at c ^ (m & 7)).
                int gg, h0;
                bool has1;
                hp.map(w.pair, &gg, &h0, &has1);
#pragma unroll 1
                for (int cc = 0; cc < N / 32; ++cc, ++q) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + as * N + cc * 32, r);
                    float* buf = s_out + (q & 1) * (32 * 128);
                    if (m == 0) bulk_wait_group_read<1>();   // the store of two boxes ago is read
                    named_bar_sync(2, 128);
                    float4* b4 = reinterpret_cast<float4*>(buf) + m * 8;
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        b4[c4 ^ (m & 7)] = make_float4(__uint_as_float(r[4 * c4]), __uint_as_float(r[4 * c4 + 1]),
                                                       __uint_as_float(r[4 * c4 + 2]), __uint_as_float(r[4 * c4 + 3]));
                    fence_proxy_async_smem();
                    if (cc == N / 32 - 1) tc_fence_before();
                    named_bar_sync(2, 128);
                    if (m == 0) {
                        if (cc == N / 32 - 1) mbar_arrive(&bars[BAR_ACCEMPTY + as]);
                        // the pair's 128 rows as one box; a phantom's half is not stored
                        if (has1) tma_store_3d(&tmS, buf, cc * 32, h0 * 64, (int)(w.b * T + w.c));
                        else tma_store_3d(&tmS1, buf, cc * 32, h0 * 64, (int)(w.b * T + w.c));
                        bulk_commit_group();
                    }
                }
            }
        }
        if (m == 0) bulk_wait_group<0>();        // stores done before the CTA leaves
        if (fail) s_flag[0] = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 13 * 32) {
        mbar_wait(&bars[BAR_DRAIN], 0, status);  // every MMA of this CTA has completed
    } else if (s_flag[0] && tid == 12 * 32) {
        // A wait gave up somewhere: give outstanding TMA loads a last (bounded)
        // chance to land before the shared memory goes away.
        const uint32_t issued = s_cnt[0], nb = s_cnt[1];
        if (nb) mbar_wait(&bars[BAR_B], (nb - 1) & 1, status);
        for (uint32_t s = 0; s < (uint32_t)kRing; ++s) {
            const uint32_t uses = issued / kRing + (s < issued % kRing ? 1u : 0u);
            if (uses) mbar_wait(&bars[BAR_XFULL + s], (uses - 1) & 1, status);
        }
    }
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, S::kTmemCols);
    }
}

template <int Q, int N>
cudaError_t launch_impl(const void* x, const float* dt, const float* A, const void* B,
                        float* states, float* logdecay, const Dims& d, int ksplit, bool rev,
                        int pc, cudaStream_t s) {
    using S = StateSmem<Q, N>;
    CUtensorMap tmX, tmB, tmS, tmS1;
    // x: pc columns a (virtual) head; a 64-column box reads zeros past them
    const uint64_t xdims[4] = {(uint64_t)pc, (uint64_t)d.H, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t xstr[3] = {(uint64_t)pc * 2, (uint64_t)(d.H * pc * 2), (uint64_t)(d.L * d.H * pc * 2)};
    const uint32_t xbox[4] = {64, 1, kStageTok, 1};
    cudaError_t e = make_tmap_bf16(&tmX, x, 4, xdims, xstr, xbox);
    if (e != cudaSuccess) return e;
    const uint64_t bdims[4] = {(uint64_t)N, (uint64_t)d.G, (uint64_t)d.L, (uint64_t)d.b};
    const uint64_t bstr[3] = {(uint64_t)N * 2, (uint64_t)(d.G * N * 2), (uint64_t)(d.L * d.G * N * 2)};
    const uint32_t bbox[4] = {64, 1, Q, 1};
    e = make_tmap_bf16(&tmB, B, 4, bdims, bstr, bbox);
    if (e != cudaSuccess) return e;
    {
        // states as rows (head, p) of N fp32 per (batch, chunk); N = 128: boxes of
        // 32 rows x 128 (plain), N = 64: boxes of 128 (or 64) rows x 32 (128-byte swizzle)
        const uint64_t sdims[3] = {(uint64_t)N, (uint64_t)(d.H * 64), (uint64_t)(d.b * d.T)};
        const uint64_t sstr[2] = {(uint64_t)N * 4, (uint64_t)(d.H * 64 * N * 4)};
        const uint32_t sbox128[3] = {128, 32, 1}, sbox64[3] = {32, 128, 1}, sbox64h[3] = {32, 64, 1};
        e = make_tmap_f32_plain(&tmS, states, 3, sdims, sstr, N == 128 ? sbox128 : sbox64, N != 128);
        if (e != cudaSuccess) return e;
        // N = 64, a head paired with a phantom: its 64 rows alone
        e = make_tmap_f32_plain(&tmS1, states, 3, sdims, sstr, N == 128 ? sbox128 : sbox64h, N != 128);
        if (e != cudaSuccess) return e;
    }
    const sm100::WaitCtx status = make_wait_ctx();
    if (!status.word) return cudaErrorUnknown;

    const int64_t items = d.b * d.T * d.G * HeadPairs((int)d.H, (int)d.G).per_group();
    if (items == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t grid = items < sms ? items : sms;
    e = cudaFuncSetAttribute(chunk_state_tc_kernel<Q, N>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
    if (e != cudaSuccess) return e;
    chunk_state_tc_kernel<Q, N><<<(unsigned)grid, kThreads, S::kAlloc, s>>>(
        tmX, tmB, tmS, tmS1, dt, A, states, logdecay, d.L, (int)d.H, (int)d.G, d.T, items, ksplit,
        rev ? 1 : 0, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_state_tc(const void* x, const float* dt, const float* A, const void* B,
                                  float* states, float* logdecay, const Dims& d, cudaStream_t s,
                                  bool rev) {
    int k = 1;
    const Dims v = virtual_heads(d, &k);
    if (v.Q == 256 && v.N == 128) return launch_impl<256, 128>(x, dt, A, B, states, logdecay, v, k, rev, head_cols(d), s);
    if (v.Q == 256 && v.N == 64) return launch_impl<256, 64>(x, dt, A, B, states, logdecay, v, k, rev, head_cols(d), s);
    if (v.Q == 128 && v.N == 128) return launch_impl<128, 128>(x, dt, A, B, states, logdecay, v, k, rev, head_cols(d), s);
    if (v.Q == 128 && v.N == 64) return launch_impl<128, 64>(x, dt, A, B, states, logdecay, v, k, rev, head_cols(d), s);
    return cudaErrorNotSupported;
}

}  // namespace ssd
