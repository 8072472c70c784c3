// tc_kernels.h -- tcgen05 (5th-generation tensor core) kernels of the chunked
// SSD forward for bf16 inputs.
#pragma once
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {

// True when the tensor-core kernels cover these sizes and dtype.
bool tc_supported(const Dims& d, Elt t);

cudaError_t launch_chunk_state_tc(const void* x, const float* dt, const float* A, const void* B,
                                  float* states, float* logdecay, const Dims& d, cudaStream_t s);
// Chunk states and the inter-chunk recurrence fused: one CTA per (batch,
// head pair) walks the chunks; writes the entering states (bf16, layout
// (b, T, H, P, N)) and the final state (fp32, nullable).
cudaError_t launch_state_walk_tc(const void* x, const float* dt, const float* A, const void* B,
                                 const float* init, void* prev, float* final_states,
                                 const Dims& d, cudaStream_t s);
// True when the forward runs the walk: enough (batch, head pair) walkers.
bool walk_preferred(const Dims& d);

cudaError_t launch_chunk_out_tc(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, const void* prev, void* y,
                                const Dims& d, cudaStream_t s);

}  // namespace ssd
