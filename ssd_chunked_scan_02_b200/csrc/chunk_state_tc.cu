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
// Per head pair the MMA is M = 128 (two heads x P = 64 rows), N = dstate,
// K = chunk: A = the two heads' scaled x tiles (MN-major), B = the chunk's
// B tile (MN-major), D in TMEM.  TMA brings x and B into 128-byte-swizzled
// shared memory; the B tile is loaded once per CTA and reused by every head
// pair; x tiles are double-buffered so the next pair's load overlaps the
// current pair's work.  The x tile is scaled in place by w_j (so the MMA
// sees bf16(w_j x_j)), the MMA runs, and the epilogue streams S to HBM
// (fp32, layout (b, T, H, P, N)).
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

template <int Q, int N>
struct StateSmem {
    static constexpr int kXTile = Q * 128;                 // one head's x tile (Q rows x 64 bf16)
    static constexpr int kB = 0;                           // N/64 blocks of Q rows x 128 B
    static constexpr int kBBytes = (N / 64) * Q * 128;
    static constexpr int kX = kB + kBBytes;                // [2 buffers][2 heads] x tiles
    static constexpr int kMaxHeads = 8;                    // 2 x up to 4 head pairs
    static constexpr int kDt = kX + 4 * kXTile;            // float [kMaxHeads][Q]: dt
    static constexpr int kW = kDt + kMaxHeads * Q * 4;     // float [kMaxHeads][Q]: w_j
    static constexpr int kBar = kW + kMaxHeads * Q * 4;    // 5 mbarriers
    static constexpr int kTmem = kBar + 8 * 8;
    static constexpr int kAbort = kTmem + 4;
    static constexpr int kTotal = kAbort + 4;
    static constexpr int kAlloc = kTotal + 1024;           // slack to align the base to 1 KB
    static constexpr uint32_t kTmemCols = (2 * N <= 128) ? 128 : 256;   // two fp32 D buffers
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
                      unsigned int* status) {
    using S = StateSmem<Q, N>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sB = smem + S::kB;
    uint8_t* sX = smem + S::kX;
    float* s_dt = reinterpret_cast<float*>(smem + S::kDt);
    float* s_w = reinterpret_cast<float*>(smem + S::kW);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);   // 0: B, 1-2: x, 3-4: MMA
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::kTmem);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + S::kAbort);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bt = blockIdx.x;
    const int64_t c = bt % T, b = bt / T;
    const int pair0 = blockIdx.y * HP;
    const int g = (2 * pair0) / (H / G);
    const int64_t t0 = c * Q;
    const int len = (int)((L - t0) < Q ? (L - t0) : Q);

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        *s_abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmB);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    // Thread 0 issues every TMA load and MMA; it also tracks what is in
    // flight so that an abort can drain it before TMEM is freed.
    bool b_pending = false;
    int x_pending[2] = {-1, -1};    // parity of an issued, not yet consumed x load
    int m_pending[2] = {-1, -1};    // parity of a committed, not yet waited MMA group
    int x_issues[2] = {0, 0};

    auto issue_x = [&](int pi) {
        const int buf = pi & 1;
        const int h0 = 2 * (pair0 + pi);
        mbar_expect_tx(&bars[1 + buf], 2 * S::kXTile);
        tma_load_4d(sX + (2 * buf + 0) * S::kXTile, &tmX, &bars[1 + buf], 0, h0, (int)t0, (int)b);
        tma_load_4d(sX + (2 * buf + 1) * S::kXTile, &tmX, &bars[1 + buf], 0, h0 + 1, (int)t0,
                    (int)b);
        x_pending[buf] = x_issues[buf] & 1;
        x_issues[buf]++;
    };

    if (tid == 0) {
        mbar_expect_tx(&bars[0], S::kBBytes);
#pragma unroll
        for (int nb = 0; nb < N / 64; ++nb)
            tma_load_4d(sB + nb * Q * 128, &tmB, &bars[0], nb * 64, g, (int)t0, (int)b);
        b_pending = true;
        issue_x(0);
        if (HP > 1) issue_x(1);
    }

    // (a0) dt of every head of the CTA for the whole chunk, in one coalesced
    // pass (heads of a token are contiguous), then per head the inclusive
    // prefix sum of dt*A (warp shuffles) and w_j = exp(cs_last - cs_j) dt_j.
    const int nh = 2 * HP;
    for (int e = tid; e < nh * Q; e += kThreads) {
        const int j = e / nh, k = e - j * nh;
        s_dt[k * Q + j] = (j < len) ? dt[(b * L + t0 + j) * H + 2 * pair0 + k] : 0.f;
    }
    __syncthreads();
    for (int k = warp; k < nh; k += kThreads / 32) {
        const float Ah = A[2 * pair0 + k];
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
    __syncthreads();

    constexpr uint32_t kIdesc = idesc_bf16_f32(128, N, /*a_mn=*/true, /*b_mn=*/true);
    bool aborted = false;

    for (int pi = 0; pi < HP; ++pi) {
        const int buf = pi & 1;
        const uint32_t use_parity = (uint32_t)((pi >> 1) & 1);

        if (pi == 0) {
            if (!mbar_wait(&bars[0], 0, status)) *s_abort = 1;
        }
        if (!mbar_wait(&bars[1 + buf], use_parity, status)) *s_abort = 1;
        __syncthreads();
        if (*s_abort) { aborted = true; break; }
        if (tid == 0) { b_pending = false; x_pending[buf] = -1; }

        // (a2, operand prep) scale each x row j of both heads by w_j, in place.
        for (int r = tid; r < 2 * Q; r += kThreads) {
            const int k = r / Q, j = r - k * Q;
            const float wj = s_w[(2 * pi + k) * Q + j];
            uint4* row = reinterpret_cast<uint4*>(sX + (2 * buf + k) * S::kXTile + j * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint4 v = row[q];
                uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162*>(&u[e]);
                    const float2 f = __bfloat1622float2(h2);
                    u[e] = pack_bf16x2(f.x * wj, f.y * wj);
                }
                row[q] = v;
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // (a2) one MMA group: D[buf] = Xw^T B over K = Q tokens.
        if (tid == 0) {
            tc_fence_after();
            const uint32_t a0 = smem_u32(sX + (2 * buf) * S::kXTile);
            const uint32_t b0 = smem_u32(sB);
#pragma unroll
            for (int ks = 0; ks < Q / 16; ++ks) {
                const uint64_t ad = smem_desc_sw128(a0 + ks * 2048, S::kXTile, 1024);
                const uint64_t bd = smem_desc_sw128(b0 + ks * 2048, Q * 128, 1024);
                mma_ss(tmem + buf * N, ad, bd, kIdesc, ks > 0);
            }
            mma_commit(&bars[3 + buf]);
            m_pending[buf] = (int)use_parity;
        }
        if (!mbar_wait(&bars[3 + buf], use_parity, status)) *s_abort = 1;
        tc_fence_after();
        __syncthreads();
        if (*s_abort) { aborted = true; break; }
        if (tid == 0) {
            m_pending[buf] = -1;
            if (pi + 2 < HP) issue_x(pi + 2);   // buffer `buf` is free again
        }

        // epilogue: row m of D = (head m / 64, p = m % 64); 32 columns at a time.
        {
            const int m = tid;
            const int h = 2 * (pair0 + pi) + (m >> 6);
            const int p = m & 63;
            float* out = states + (((b * T + c) * H + h) * 64 + p) * (int64_t)N;
            const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
#pragma unroll
            for (int cc = 0; cc < N / 32; ++cc) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_base + buf * N + cc * 32, r);
                float4* o4 = reinterpret_cast<float4*>(out + cc * 32);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    o4[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                        __uint_as_float(r[4 * q + 2]),
                                        __uint_as_float(r[4 * q + 3]));
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    if (aborted && tid == 0) {
        // Drain what is still in flight (bounded) before the shared memory and
        // TMEM go away.
        if (b_pending) mbar_wait(&bars[0], 0, status);
        for (int k = 0; k < 2; ++k) {
            if (x_pending[k] >= 0) mbar_wait(&bars[1 + k], (uint32_t)x_pending[k], status);
            if (m_pending[k] >= 0) mbar_wait(&bars[3 + k], (uint32_t)m_pending[k], status);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, S::kTmemCols);
    }
}

int pick_pairs_per_cta(int64_t H, int64_t G) {
    const int64_t pairs_in_group = (H / G) / 2;
    for (int hp = 4; hp > 1; --hp)
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
    unsigned int* status = device_status_ptr();
    if (!status) return cudaErrorUnknown;

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
