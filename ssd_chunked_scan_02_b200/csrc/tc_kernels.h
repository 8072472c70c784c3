// tc_kernels.h -- tcgen05 (5th-generation tensor core) kernels of the chunked
// SSD forward for bf16 inputs.
#pragma once
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {

// The tcgen05 kernels work on heads of headdim 64.  A head of headdim 64 k is
// handled as k such (virtual) heads that share dt, A and D -- the rows of a
// state evolve independently, and x, y and the states (b, ., H, P, .) are
// the same memory as (b, ., H k, 64, .).  A head of headdim 32 runs as a head
// of 64 whose last 32 rows are zero: its x tiles are loaded with zeros past
// column 32 (the tensor map's edge), y tiles are stored up to column 32, the
// kernels' own state buffers keep 64 rows, and states in the caller's
// (b, H, 32, N) layout are read and written row by row.  Returns the virtual
// sizes (H k, P 64) and k.
inline Dims virtual_heads(const Dims& d, int* ksplit) {
    Dims v = d;
    *ksplit = d.P >= 64 ? (int)(d.P / 64) : 1;
    v.H = d.H * *ksplit;
    v.P = 64;
    return v;
}
// Columns of x (and y) per virtual head, and the rows per head of the
// internal state buffers, for a head of the caller's headdim.
inline int head_cols(const Dims& d) { return d.P < 64 ? (int)d.P : 64; }
inline int64_t state_rows(int64_t P) { return P < 64 ? 64 : P; }

// The state kernels work on pairs of (virtual) heads of one group.  A group
// with an odd number of heads pairs its last head with a phantom: its x is
// read as zeros (an out-of-range head coordinate) and its outputs are not
// written.
struct HeadPairs {
    int hpg, ppg;      // heads and pairs per group
    __host__ __device__ explicit HeadPairs(int H, int G) : hpg(H / G), ppg((H / G + 1) / 2) {}
    __host__ __device__ int per_group() const { return ppg; }
    // pair -> its group, first head, and whether the second head exists
    __host__ __device__ void map(int pair, int* g, int* h0, bool* has1) const {
        *g = pair / ppg;
        const int l = pair - *g * ppg;
        *h0 = *g * hpg + 2 * l;
        *has1 = 2 * l + 1 < hpg;
    }
};

// True when the tensor-core kernels cover these sizes and dtype (headdim 32
// or 64 k up to 256; the step entry points, whose state buffers are the
// caller's, take the multiples of 64 only).
bool tc_supported(const Dims& d, Elt t);

// rev: the backward's per-chunk dL/dh contributions instead (weights
// exp(cs_j); pass dy as x and C as B).
cudaError_t launch_chunk_state_tc(const void* x, const float* dt, const float* A, const void* B,
                                  float* states, float* logdecay, const Dims& d, cudaStream_t s,
                                  bool rev = false);
// Chunk states and the inter-chunk recurrence fused: one CTA per (batch,
// head pair) walks the chunks; writes the entering states (bf16, layout
// (b, T, H, P, N)) and the final state (fp32, nullable).
cudaError_t launch_state_walk_tc(const void* x, const float* dt, const float* A, const void* B,
                                 const float* init, void* prev, float* final_states,
                                 const Dims& d, cudaStream_t s);
// True when the forward runs the walk: enough (batch, head pair) walkers.
bool walk_preferred(const Dims& d);

// The whole forward in one launch (walkers of two or four heads and output
// tiles side by side; walk_out_tc.cu): dstate 64 or 128, chunk 128 or 256.
// `sched` is device scratch of walk_out_sched_bytes(d) bytes (zeroed by the
// launcher on `s`); prev as for the walk.
bool walk_out_supported(const Dims& d);
// ... and the forward takes it (enough chunks for the overlap to pay).
bool walk_out_preferred(const Dims& d);
size_t walk_out_sched_bytes(const Dims& d);
cudaError_t launch_walk_out_tc(const void* x, const float* dt, const float* A, const void* B,
                               const void* C, const float* D, const float* init, void* prev,
                               void* y, float* final_states, int* sched, const Dims& d,
                               cudaStream_t s);

cudaError_t launch_chunk_out_tc(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, const void* prev, void* y,
                                const Dims& d, cudaStream_t s);

}  // namespace ssd
