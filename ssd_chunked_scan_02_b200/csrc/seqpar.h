// seqpar.h -- launchers of the sequence-parallel pieces (seqpar.cu,
// state_apply_tc.cu).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {

constexpr int kSeqparTile = 128;    // tokens per correction tile

cudaError_t launch_seq_logdecay(const float* dt, const float* A, float* out, const Dims& d,
                                cudaStream_t s);
cudaError_t launch_state_combine(const float* F, const float* ld, const float* init, float* out,
                                 int rank, const Dims& d, cudaStream_t s);
// Number of 128-token correction tiles of the shard.
int64_t correction_tiles(const Dims& d);
// Per (batch, head): tile_prefix (b, ntiles, H) = exclusive prefix of dt*A
// over tiles (log2 units), final += exp(Lambda) h_in (fin nullable), h_in
// rounded to bf16 into h_bf16 (nullable).
cudaError_t launch_correction_prep(const float* h_in, const float* dt, const float* A,
                                   float* tile_prefix, float* fin, __nv_bfloat16* h_bf16,
                                   const Dims& d, cudaStream_t s);
cudaError_t launch_correction_simt(const float* h_in, const float* dt, const float* A,
                                   const void* C, const float* tile_prefix, void* y,
                                   const Dims& d, Elt t, cudaStream_t s);
// tcgen05 correction (bf16, headdim a multiple of 64 up to 256, dstate 64 or 128).
bool correction_tc_supported(const Dims& d, Elt t);
cudaError_t launch_correction_tc(const __nv_bfloat16* h_bf16, const float* dt, const float* A,
                                 const void* C, const float* tile_prefix, void* y, const Dims& d,
                                 cudaStream_t s);

}  // namespace ssd
