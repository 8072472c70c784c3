// state_walk_body.cuh -- one walker of the fused chunk-state recurrence
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
// A walker is one CTA that owns HP (virtual) heads of one (batch, group) and
// walks the chunks in order; S_c never leaves the chip.  HP = 2 is the
// standalone walk kernel (two walkers fit an SM); HP = 4 (dstate 128 only)
// is the walker role of the fused walk + output kernel, which holds an SM on
// its own.  Tensor memory holds two fp32 tiles: the running state h and the
// chunk's accumulator S.  The MMAs of chunk c write S from zero; the
// epilogue warps then read h and S, form h' = exp(cs_last) h + S, store h'
// back over h and write it out as the state entering chunk c + 1 (bf16), or
// as the final state (fp32) after the last chunk.  The MMAs of chunk c + 1
// wait only until the epilogue has read S, not for its stores, so the loads,
// scaling and MMAs of the next chunk stream while the epilogue works.
//
// With dstate N = 128 the MMA forms S^T (M = 128 state rows n, N = HP heads x
// P = 64), so a TMEM lane is a state column and a warp's prev/final stores are
// contiguous along n; with N = 64 (HP = 2) it forms S (M = two heads x P rows,
// N = 64), a lane is a (head, p) row.  x and B come by TMA in 64-token
// sub-steps through a three-entry ring; x rows are scaled in place by the
// decay weights w_j = exp(cs_last - cs_j) dt_j before the MMA reads them.
//
// Roles (32 (2 HP + 6) threads): warps 0 .. 2HP-1 dt prefix sums (warp =
// (head, half of the chunk)) and x scaling (thread t scales row t of each
// ring entry: head t / 64, token t % 64, and each warp reports its rows by
// its own arrival); the next four warps the state epilogue; then the TMA
// producer and the MMA issuer (TMEM owner).  Warps past these (a walker run
// by a larger block) only take part in the block's barriers.  Every wait is
// bounded; a warpgroup leaves its loop only when all its threads agree
// (bar.red.or).
//
// When `progress` is given (the walker of four heads), the walker publishes
// how many entering states are in global memory (c + 1 once prev_c is
// written) for consumers in other CTAs of the same launch.  The epilogue
// warps meet after their stores and one of them release-stores the count
// into shared memory; lane 1 of the producer warp, otherwise idle, acquires
// it there and release-stores it to `progress` (release and acquire are
// cumulative, so a consumer that acquires the count sees every epilogue
// thread's stores).  The epilogue never waits for global memory.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace ssd {
namespace walk {
using namespace sm100;

// Split forms for software pipelining: a TMEM load without its wait, the wait
// that orders every later use of the loaded registers (they are its in/out
// operands, so no use can be scheduled above it), a TMEM store without its
// wait (the source registers are read when the store issues; later
// instructions may reuse them) and the wait for all of this thread's stores.
__device__ __forceinline__ void tmem_ld32x2_nowait(uint32_t ta, uint32_t tb, uint32_t (&ra)[32],
                                                   uint32_t (&rb)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];"
        : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]),
          "=r"(ra[6]), "=r"(ra[7]), "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]),
          "=r"(ra[12]), "=r"(ra[13]), "=r"(ra[14]), "=r"(ra[15]), "=r"(ra[16]), "=r"(ra[17]),
          "=r"(ra[18]), "=r"(ra[19]), "=r"(ra[20]), "=r"(ra[21]), "=r"(ra[22]), "=r"(ra[23]),
          "=r"(ra[24]), "=r"(ra[25]), "=r"(ra[26]), "=r"(ra[27]), "=r"(ra[28]), "=r"(ra[29]),
          "=r"(ra[30]), "=r"(ra[31]), "=r"(rb[0]), "=r"(rb[1]), "=r"(rb[2]), "=r"(rb[3]),
          "=r"(rb[4]), "=r"(rb[5]), "=r"(rb[6]), "=r"(rb[7]), "=r"(rb[8]), "=r"(rb[9]),
          "=r"(rb[10]), "=r"(rb[11]), "=r"(rb[12]), "=r"(rb[13]), "=r"(rb[14]), "=r"(rb[15]),
          "=r"(rb[16]), "=r"(rb[17]), "=r"(rb[18]), "=r"(rb[19]), "=r"(rb[20]), "=r"(rb[21]),
          "=r"(rb[22]), "=r"(rb[23]), "=r"(rb[24]), "=r"(rb[25]), "=r"(rb[26]), "=r"(rb[27]),
          "=r"(rb[28]), "=r"(rb[29]), "=r"(rb[30]), "=r"(rb[31])
        : "r"(ta), "r"(tb)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld64(uint32_t (&ra)[32], uint32_t (&rb)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(ra[0]), "+r"(ra[1]), "+r"(ra[2]), "+r"(ra[3]), "+r"(ra[4]), "+r"(ra[5]),
                   "+r"(ra[6]), "+r"(ra[7]), "+r"(ra[8]), "+r"(ra[9]), "+r"(ra[10]),
                   "+r"(ra[11]), "+r"(ra[12]), "+r"(ra[13]), "+r"(ra[14]), "+r"(ra[15]),
                   "+r"(ra[16]), "+r"(ra[17]), "+r"(ra[18]), "+r"(ra[19]), "+r"(ra[20]),
                   "+r"(ra[21]), "+r"(ra[22]), "+r"(ra[23]), "+r"(ra[24]), "+r"(ra[25]),
                   "+r"(ra[26]), "+r"(ra[27]), "+r"(ra[28]), "+r"(ra[29]), "+r"(ra[30]),
                   "+r"(ra[31]), "+r"(rb[0]), "+r"(rb[1]), "+r"(rb[2]), "+r"(rb[3]), "+r"(rb[4]),
                   "+r"(rb[5]), "+r"(rb[6]), "+r"(rb[7]), "+r"(rb[8]), "+r"(rb[9]), "+r"(rb[10]),
                   "+r"(rb[11]), "+r"(rb[12]), "+r"(rb[13]), "+r"(rb[14]), "+r"(rb[15]),
                   "+r"(rb[16]), "+r"(rb[17]), "+r"(rb[18]), "+r"(rb[19]), "+r"(rb[20]),
                   "+r"(rb[21]), "+r"(rb[22]), "+r"(rb[23]), "+r"(rb[24]), "+r"(rb[25]),
                   "+r"(rb[26]), "+r"(rb[27]), "+r"(rb[28]), "+r"(rb[29]), "+r"(rb[30]),
                   "+r"(rb[31])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_st32_nowait(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
                   "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
                   "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
                   "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
                   "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]),
                   "r"(r[31])
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

constexpr int kSub = 64;                 // tokens per ring entry
constexpr int kPrefetch = 6;             // L2 prefetch distance, in ring entries

template <int HP>
struct Roles {
    static constexpr int kPW = 2 * HP;             // prefix / scale warps
    static constexpr int kEpi = kPW;               // first of the four epilogue warps
    static constexpr int kProd = kPW + 4;          // TMA producer warp
    static constexpr int kMma = kPW + 5;           // MMA issuer and TMEM owner
    static constexpr int kThreads = 32 * (kPW + 6);
};

template <int Q, int N, int HP>
struct Smem {
    // ring entries of 64 tokens (HP heads' x rows and B's N/64 blocks)
    static constexpr int kStages = 3;
    // one chunk accumulator: the next chunk's MMAs wait only until the
    // epilogue has read it (two measured no faster for N = 64)
    static constexpr int kSSlots = 1;
    static constexpr int kXPart = HP * kSub * 128;         // HP heads x 64 rows x 128 B
    static constexpr int kBPart = (N / 64) * kSub * 128;   // N/64 blocks x 64 rows x 128 B
    static constexpr int kEntry = kXPart + kBPart;
    static constexpr int kRing = 0;
    static constexpr int kW = kRing + kStages * kEntry;    // float [2 buf][HP heads][Q]: w_j
    static constexpr int kA = kW + 2 * HP * Q * 4;         // float [2 buf][HP]: chunk decays
    static constexpr int kSeg = kA + 2 * HP * 4;           // float [2 buf][2 HP]: segment sums
    static constexpr int kBar = kSeg + 2 * 2 * HP * 4;
    static constexpr int kTmem = kBar + 24 * 8;
    static constexpr int kFlags = kTmem + 16;
    static constexpr int kTotal = kFlags + 16;
    static constexpr int kAlloc = kTotal + 1024;
    // TMEM: the running state h, then the chunk accumulator S
    static constexpr uint32_t kCols = (N == 128) ? 64 * HP : 64;   // columns of one tile
    static constexpr uint32_t kColH = 0;
    static constexpr uint32_t kColS = kCols;
    static constexpr uint32_t kTmemCols = 2 * kCols;
    static_assert(N == 128 || HP == 2, "dstate 64 walks two heads (M = 128 rows)");
    static_assert(kAlloc <= 232448, "shared memory");
    static_assert(kTmemCols <= 512, "TMEM");
};

enum {
    BAR_FULL = 0,        // 4: ring entry loaded (TMA transaction count)
    BAR_EMPTY = 4,       // 4: ring entry read by the MMAs
    BAR_SCALED = 8,      // 4: ring entry's x rows scaled (2 HP warp arrivals)
    BAR_AREADY = 12,     // 2: chunk decays of buffer cb published
    BAR_AFREE = 14,      // 2: the epilogue has read buffer cb's decays
    BAR_SFULL = 16,      // 2: the chunk's MMAs into accumulator slot s have completed
    BAR_SEMPTY = 18,     // 2: the epilogue has read accumulator slot s
    BAR_COUNT = 20
};

// One walker: heads h0 .. h0 + HP - 1 of group g in batch b, of which the
// first `nreal` exist (the others are phantoms: their x is read out of range,
// as zeros, and nothing of theirs is written).  H counts virtual heads
// (headdim 64); real head = virtual head / ksplit.  `smem` is 1024-aligned.
// progress: where the count of entering states written is published, or
// nullptr.
template <int Q, int N, int HP>
__device__ __forceinline__ void body(const CUtensorMap* tmX, const CUtensorMap* tmB,
                                     const float* __restrict__ dt, const float* __restrict__ A,
                                     const float* __restrict__ init,
                                     __nv_bfloat16* __restrict__ prev, float* __restrict__ fin,
                                     int64_t L, int H, int G, int64_t T, int ksplit, int pcols,
                                     int64_t b, int g, int h0, int nreal, uint8_t* smem,
                                     int* progress, const WaitCtx& status) {
    using S = Smem<Q, N, HP>;
    using R = Roles<HP>;
    constexpr bool kTrans = (N == 128);
    constexpr int kNSub = Q / kSub;
    constexpr int kStages = S::kStages;
    constexpr int kSSlots = S::kSSlots;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hr = H / ksplit;

    uint8_t* ring = smem + S::kRing;
    float* s_w = reinterpret_cast<float*>(smem + S::kW);
    float* s_a = reinterpret_cast<float*>(smem + S::kA);
    float* s_seg = reinterpret_cast<float*>(smem + S::kSeg);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + S::kFlags);

    if (tid == 0) {
        for (int i = 0; i < BAR_COUNT; ++i)
            mbar_init(&bars[i], (i >= BAR_SCALED && i < BAR_SCALED + kStages) ? R::kPW : 1);
        s_flag[0] = 0;
        s_flag[1] = 0;                              // entering states written (count)
        fence_mbar_init();
    }
    if (warp == R::kMma) {
        tmem_alloc(s_tmem, S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int64_t nsteps = T * kNSub;

    if (warp == R::kProd) {
        // ================================================== TMA producer
        if (lane == 0) {
            prefetch_tmap(tmX);
            prefetch_tmap(tmB);
            bool ok = true;
            for (int64_t si = 0; si < nsteps && ok; ++si) {
                const int e = (int)(si % kStages);
                const int64_t u = si / kStages;
                if (u >= 1) ok = mbar_wait(&bars[BAR_EMPTY + e], (uint32_t)((u - 1) & 1), status);
                if (!ok) break;
                const int row = (int)((si / kNSub) * Q + (si % kNSub) * kSub);
                uint8_t* ent = ring + e * S::kEntry;
                mbar_expect_tx(&bars[BAR_FULL + e], S::kEntry);
#pragma unroll
                for (int k = 0; k < HP; ++k)     // a phantom's x is read out of range: zeros
                    tma_load_4d(ent + k * kSub * 128, tmX, &bars[BAR_FULL + e], 0,
                                k < nreal ? h0 + k : H, row, (int)b);
                for (int nb = 0; nb < N / 64; ++nb)
                    tma_load_4d(ent + S::kXPart + nb * kSub * 128, tmB, &bars[BAR_FULL + e],
                                nb * 64, g, row, (int)b);
                // the boxes six entries on into L2, so that their loads (issued when
                // a ring entry frees) find them there
                if (si + kPrefetch < nsteps) {
                    const int rp = (int)(((si + kPrefetch) / kNSub) * Q + ((si + kPrefetch) % kNSub) * kSub);
#pragma unroll
                    for (int k = 0; k < HP; ++k)
                        if (k < nreal) tma_prefetch_4d(tmX, 0, h0 + k, rp, (int)b);
                    for (int nb = 0; nb < N / 64; ++nb) tma_prefetch_4d(tmB, nb * 64, g, rp, (int)b);
                }
            }
            if (!ok) s_flag[0] = 1;
        } else if (lane == 1 && progress) {
            // publisher: forwards the epilogue's count (monotone) to global memory.
            // The last count is T (1 after the initial state, c + 2 after chunk c
            // for c < T - 1).  Gives up when a role of the walker has, or after
            // about a second without news.
            int last = 0;
            uint64_t t0 = global_ns();
            while (last < (int)T) {
                const int v = ld_acquire_cta_smem(&s_flag[1]);
                if (v > last) {
                    st_release_gpu(progress, v);
                    last = v;
                    t0 = global_ns();
                    continue;
                }
                if (s_flag[0] || *reinterpret_cast<volatile unsigned int*>(status.word) == status.token)
                    break;
                if (global_ns() - t0 > kWaitLimitNs) {
                    atomicExch(status.word, status.token);
                    break;
                }
                __nanosleep(64);
            }
        }
    } else if (warp == R::kMma) {
        // ================================================== MMA issuer
        if (lane == 0) {
            // N = 128: S^T (M = 128 state rows, N = 64 HP head columns) = B^T (w x)
            // N = 64:  S   (M = 128 pair rows,  N = 64 state columns) = (w x)^T B
            constexpr uint32_t kIdesc = idesc_bf16_f32(128, kTrans ? 64 * HP : N, true, true);
            bool ok = true;
            int64_t si = 0;
            for (int64_t c = 0; c < T && ok; ++c) {
                // accumulator slot sl is free once the epilogue has read the S of
                // chunk c - kSSlots
                const int sl = (int)(c % kSSlots);
                const uint32_t dS = tmem + S::kColS + sl * S::kCols;
                if (c >= kSSlots)
                    ok = mbar_wait(&bars[BAR_SEMPTY + sl], (uint32_t)(((c / kSSlots) - 1) & 1), status);
                for (int sub = 0; sub < kNSub && ok; ++sub, ++si) {
                    const int e = (int)(si % kStages);
                    const int64_t u = si / kStages;
                    ok = mbar_wait(&bars[BAR_SCALED + e], (uint32_t)(u & 1), status);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t x0 = smem_u32(ring + e * S::kEntry);
                    const uint32_t b0 = x0 + S::kXPart;
#pragma unroll
                    for (int ks = 0; ks < kSub / 16; ++ks) {
                        // x: HP 64-column atoms (heads) 8 KB apart; B: 64-column
                        // atoms of dstate 8 KB apart; 8-row groups 1024 B apart.
                        const uint64_t xd = smem_desc_sw128(x0 + ks * 2048, kSub * 128, 1024);
                        const uint64_t bd = smem_desc_sw128(b0 + ks * 2048, kSub * 128, 1024);
                        const bool acc = (sub | ks) != 0;
                        if (kTrans) mma_ss(dS, bd, xd, kIdesc, acc);
                        else mma_ss(dS, xd, bd, kIdesc, acc);
                    }
                    mma_commit(&bars[BAR_EMPTY + e]);
                }
                if (ok) mma_commit(&bars[BAR_SFULL + sl]);
            }
            if (!ok) s_flag[0] = 1;
        }
    } else if (warp < R::kPW) {
        // ================================================== dt prefix sums and x scaling
        // Warp w: head hk = w / 2 of the walker, half sg = w % 2 of the chunk; lane
        // holds kPer consecutive tokens' dt, loaded one chunk ahead.
        constexpr int kPer = Q / 64;
        constexpr int kHalf = Q / 2;
        constexpr int kPT = 32 * R::kPW;            // threads of this role
        const int hk = warp >> 1, sg = warp & 1;
        const bool real = hk < nreal;
        const float Ak = real ? A[(h0 + hk) / ksplit] : 0.f;
        float dreg[kPer];
        auto load_dt = [&](int64_t c) {
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int64_t tok = c * Q + sg * kHalf + lane * kPer + k;
                dreg[k] = (real && tok < L) ? dt[(b * L + tok) * Hr + (h0 + hk) / ksplit] : 0.f;
            }
        };
        // w_j and the chunk decay of this head into buffer buf
        auto prefix = [&](int buf) {
            float v[kPer];
            float run = 0.f;                       // tokens past the sequence end add 0
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                run += dreg[k] * Ak;
                v[k] = run;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float uu = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += uu;
            }
            if (lane == 31) s_seg[buf * R::kPW + warp] = incl;
            named_bar_sync(1, kPT);
            const float s0 = s_seg[buf * R::kPW + hk * 2], s1 = s_seg[buf * R::kPW + hk * 2 + 1];
            const float off = (incl - run) + (sg ? s0 : 0.f);
            const float last = s0 + s1;
            float* wk = s_w + (buf * HP + hk) * Q + sg * kHalf + lane * kPer;
#pragma unroll
            for (int k = 0; k < kPer; ++k) wk[k] = expf(last - (v[k] + off)) * dreg[k];
            if (sg == 0 && lane == 0) s_a[buf * HP + hk] = expf(last);
        };
        bool fail = false;
        int64_t si = 0;
        load_dt(0);
        for (int64_t c = 0; c < T; ++c) {
            const int cb = (int)(c & 1);
            // buffer cb is free once the epilogue has read chunk c-2's decays
            if (!fail && c >= 2)
                fail = !mbar_wait(&bars[BAR_AFREE + cb], (uint32_t)(((c >> 1) - 1) & 1), status);
            prefix(cb);
            if (c + 1 < T) load_dt(c + 1);
            // publishes w_j and the decays, and shares every thread's outcome
            if (named_bar_or(1, kPT, fail)) {
                fail = true;
                break;
            }
            if (tid == 0) mbar_arrive(&bars[BAR_AREADY + cb]);
            const float* wb = s_w + cb * HP * Q;
            for (int sub = 0; sub < kNSub; ++sub, ++si) {
                const int e = (int)(si % kStages);
                const int64_t u = si / kStages;
                const bool ok = mbar_wait(&bars[BAR_FULL + e], (uint32_t)(u & 1), status);
                if (__any_sync(0xffffffffu, !ok)) {
                    fail = true;                      // shared at the next chunk's barrier
                    break;
                }
                // row tid of the entry: head tid / 64, token sub * 64 + tid % 64; its
                // 16-byte chunks are visited in a per-row rotated order (bank-conflict free)
                const int k = tid >> 6, jl = tid & 63;
                const float wj = wb[k * Q + sub * kSub + jl];
                uint4* row = reinterpret_cast<uint4*>(ring + e * S::kEntry + k * kSub * 128 + jl * 128);
                uint4 v[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] = row[q ^ (jl & 7)];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t* uw = reinterpret_cast<uint32_t*>(&v[q]);
#pragma unroll
                    for (int ee = 0; ee < 4; ++ee) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&uw[ee]));
                        uw[ee] = pack_bf16x2(f.x * wj, f.y * wj);
                    }
                    row[q ^ (jl & 7)] = v[q];
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[BAR_SCALED + e]);
            }
        }
        if (fail) s_flag[0] = 1;
    } else if (warp < R::kEpi + 4) {
        // ================================================== state epilogue (four warps)
        const int m = tid - 32 * R::kEpi;              // TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tH = tmem + lane_base + S::kColH;
        bool fail = false;
        // the entering states up to prev_{v-1} have been stored (for the publisher)
        auto publish = [&](int v) {
            if (!progress) return;
            named_bar_sync(2, 128);
            if (m == 0) st_release_cta_smem(&s_flag[1], v);
        };
        // h_{-1} = init (or zero): into the state tile, and out as chunk 0's entering state
        if (kTrans) {
            // lane m = state column n; TMEM column cc*32+e = (head cc/2, p = (cc&1)*32 + e)
            const int n = m;
#pragma unroll 1
            for (int cc = 0; cc < 2 * HP; ++cc) {
                const int k = cc >> 1, p0 = (cc & 1) * 32;
                // init: (b, H, pcols, N), pcols = 64 or 32 (rows pcols .. 63 zero)
                const int64_t srow = ((b * H + h0 + k) * pcols + p0) * (int64_t)N + n;
                const bool real = k < nreal;
                const bool rows = init && real && p0 < pcols;
                uint32_t r[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    r[e] = __float_as_uint(rows ? init[srow + (int64_t)e * N] : 0.f);
                if (real) {
                    __nv_bfloat16* pr = prev + (((b * T) * H + h0 + k) * 64 + p0) * (int64_t)N + n;
#pragma unroll
                    for (int e = 0; e < 32; ++e) pr[(int64_t)e * N] = __float2bfloat16_rn(__uint_as_float(r[e]));
                }
                uint32_t lo[16], hi[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    lo[e] = r[e];
                    hi[e] = r[16 + e];
                }
                tmem_st16(tH + cc * 32, lo);
                tmem_st16(tH + cc * 32 + 16, hi);
            }
        } else {
            // lane m = (head m / 64, p = m % 64); TMEM columns = state n (N = 64)
            const int k = m >> 6, p = m & 63;
            const bool real = k < nreal;
            const int64_t srow = ((b * H + h0 + k) * pcols + p) * (int64_t)N;
#pragma unroll 1
            for (int cc = 0; cc < N / 32; ++cc) {
                uint32_t r[32];
                if (init && real && p < pcols) {
                    const float4* s4 = reinterpret_cast<const float4*>(init + srow + cc * 32);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 f = s4[q];
                        r[4 * q] = __float_as_uint(f.x);
                        r[4 * q + 1] = __float_as_uint(f.y);
                        r[4 * q + 2] = __float_as_uint(f.z);
                        r[4 * q + 3] = __float_as_uint(f.w);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = 0u;
                }
                __nv_bfloat16* pr = prev + (((b * T) * H + h0 + k) * 64 + p) * (int64_t)N + cc * 32;
#pragma unroll
                for (int e = 0; e < 32 && real; e += 8) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));
                    v.y = pack_bf16x2(__uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
                    v.z = pack_bf16x2(__uint_as_float(r[e + 4]), __uint_as_float(r[e + 5]));
                    v.w = pack_bf16x2(__uint_as_float(r[e + 6]), __uint_as_float(r[e + 7]));
                    *reinterpret_cast<uint4*>(pr + e) = v;
                }
                uint32_t lo[16], hi[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    lo[e] = r[e];
                    hi[e] = r[16 + e];
                }
                tmem_st16(tH + cc * 32, lo);
                tmem_st16(tH + cc * 32 + 16, hi);
            }
        }
        publish(1);

        for (int64_t c = 0; c < T; ++c) {
            const int cb = (int)(c & 1);
            const int sl = (int)(c % kSSlots);
            const uint32_t tS = tmem + lane_base + S::kColS + sl * S::kCols;
            const bool last = (c + 1 == T);
            fail = !mbar_wait(&bars[BAR_AREADY + cb], (uint32_t)((c >> 1) & 1), status) ||
                   !mbar_wait(&bars[BAR_SFULL + sl], (uint32_t)((c / kSSlots) & 1), status);
            if (named_bar_or(2, 128, fail)) {
                fail = true;
                break;
            }
            tc_fence_after();
            float av[HP];
#pragma unroll
            for (int k = 0; k < HP; ++k) av[k] = s_a[cb * HP + k];
            named_bar_sync(2, 128);
            if (m == 0) mbar_arrive(&bars[BAR_AFREE + cb]);
            // pass 1: h' = a h + S in TMEM (h' over h); then S is free for the next
            // chunk.  Per 32-column block: the update in place in the loaded
            // registers, its store issued without a wait, then the next block's
            // loads; one wait for all the stores at the end.
            {
                const int nk = kTrans ? 2 * HP : N / 32;
                uint32_t hr[32], sr[32];
                tmem_ld32x2_nowait(tH, tS, hr, sr);
#pragma unroll 1
                for (int cc = 0; cc < nk; ++cc) {
                    tmem_wait_ld64(hr, sr);
                    const int k = kTrans ? (cc >> 1) : (m >> 6);
                    float a = av[0];
#pragma unroll
                    for (int kk = 1; kk < HP; ++kk) a = (k == kk) ? av[kk] : a;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        hr[e] = __float_as_uint(fmaf(a, __uint_as_float(hr[e]), __uint_as_float(sr[e])));
                    tmem_st32_nowait(tH + cc * 32, hr);
                    if (cc + 1 < nk) tmem_ld32x2_nowait(tH + (cc + 1) * 32, tS + (cc + 1) * 32, hr, sr);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            named_bar_sync(2, 128);
            if (m == 0) mbar_arrive(&bars[BAR_SEMPTY + sl]);
            // pass 2: h' out, as the state entering chunk c + 1 (bf16) or the final state
            if (last && !fin) continue;
            if (kTrans) {
                const int n = m;
#pragma unroll 1
                for (int cc = 0; cc < 2 * HP; ++cc) {
                    const int k = cc >> 1, p0 = (cc & 1) * 32;
                    if (k >= nreal) break;            // a phantom's state is not written
                    uint32_t hr[32];
                    tmem_ld32(tH + cc * 32, hr);
                    if (!last) {
                        __nv_bfloat16* pr =
                            prev + (((b * T + c + 1) * H + h0 + k) * 64 + p0) * (int64_t)N + n;
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            pr[(int64_t)e * N] = __float2bfloat16_rn(__uint_as_float(hr[e]));
                    } else if (p0 < pcols) {
                        float* fp = fin + ((b * H + h0 + k) * pcols + p0) * (int64_t)N + n;
#pragma unroll
                        for (int e = 0; e < 32; ++e) fp[(int64_t)e * N] = __uint_as_float(hr[e]);
                    }
                }
            } else {
                const int k = m >> 6, p = m & 63;
                const bool real = k < nreal;
#pragma unroll 1
                for (int cc = 0; cc < N / 32; ++cc) {
                    uint32_t hr[32];
                    tmem_ld32(tH + cc * 32, hr);
                    if (!real) continue;                  // a phantom's state is not written
                    if (!last) {
                        __nv_bfloat16* pr =
                            prev + (((b * T + c + 1) * H + h0 + k) * 64 + p) * (int64_t)N + cc * 32;
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(hr[e]), __uint_as_float(hr[e + 1]));
                            v.y = pack_bf16x2(__uint_as_float(hr[e + 2]), __uint_as_float(hr[e + 3]));
                            v.z = pack_bf16x2(__uint_as_float(hr[e + 4]), __uint_as_float(hr[e + 5]));
                            v.w = pack_bf16x2(__uint_as_float(hr[e + 6]), __uint_as_float(hr[e + 7]));
                            *reinterpret_cast<uint4*>(pr + e) = v;
                        }
                    } else if (p < pcols) {
                        float4* f4 = reinterpret_cast<float4*>(
                            fin + ((b * H + h0 + k) * pcols + p) * (int64_t)N + cc * 32);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            f4[q] = make_float4(__uint_as_float(hr[4 * q]), __uint_as_float(hr[4 * q + 1]),
                                                __uint_as_float(hr[4 * q + 2]), __uint_as_float(hr[4 * q + 3]));
                    }
                }
            }
            if (!last) publish((int)c + 2);
        }
        if (fail) s_flag[0] = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (s_flag[0] && tid == R::kProd * 32) {
        // A wait gave up somewhere: give outstanding TMA loads and MMAs a last
        // (bounded) chance to land before the shared memory and TMEM go away.
        for (int k = 0; k < kStages; ++k) mbar_wait(&bars[BAR_FULL + k], 0, status);
        for (int k = 0; k < kSSlots; ++k) mbar_wait(&bars[BAR_SFULL + k], 0, status);
    }
    __syncthreads();
    if (warp == R::kMma) {
        tc_fence_after();
        tmem_dealloc(tmem, S::kTmemCols);
    }
}

}  // namespace walk
}  // namespace ssd
