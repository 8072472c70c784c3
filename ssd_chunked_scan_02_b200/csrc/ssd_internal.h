// ssd_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

struct Dims {
    int64_t b, L, H, P, N, G;
    int Q;        // chunk size
    int64_t T;    // number of chunks = ceil(L / Q)
};

// Element type of x, B, C, y and the prev-state buffer.
enum class Elt { F32 = 0, BF16 = 1 };

// SIMT kernels (exact fp32 arithmetic; any supported size).
cudaError_t launch_chunk_state_simt(const void* x, const float* dt, const float* A, const void* B,
                                    float* states, float* logdecay, const Dims& d, Elt t,
                                    cudaStream_t s);
cudaError_t launch_chunk_out_simt(const void* x, const float* dt, const float* A, const void* B,
                                  const void* C, const float* D, const void* prev, void* y,
                                  const Dims& d, Elt t, cudaStream_t s);

// Inter-chunk recurrence (fp32), writes prev states in `t` and the final state;
// reverse: the chunks last to first (the backward's pass over dL/dh).
// p_ext (when non-zero and below d.P): init and final_states have p_ext rows
// per head ((b, H, p_ext, N)), the state buffers d.P (rows p_ext.. zero).
// prev_lo (bf16 only, nullable): also the rounding residue of each prev
// element, bf16(h - bf16(h)).
cudaError_t launch_state_pass(const float* states, const float* logdecay, const float* init,
                              void* prev, float* final_states, const Dims& d, Elt t,
                              cudaStream_t s, bool reverse = false, int64_t p_ext = 0,
                              void* prev_lo = nullptr);

// Decode step.
cudaError_t launch_step(float* state, const void* x, const float* dt, const float* A,
                        const void* B, const void* C, const float* D, void* y, const Dims& d,
                        Elt t, cudaStream_t s);

// Copies init (or zeros) into final: the L == 0 case.
cudaError_t launch_copy_or_zero(const float* init, float* final_states, int64_t n,
                                cudaStream_t s);

// Backward (gradients of the forward), exact fp32 on the CUDA cores.
size_t backward_workspace_bytes(const Dims& d);
bool backward_supported(const Dims& d);
cudaError_t launch_backward(const void* x, const float* dt, const float* A, const void* B,
                            const void* C, const float* D, const float* init, const void* dy,
                            const float* dfinal, float* dx, float* ddt, float* dA, float* dB,
                            float* dC, float* dD, float* dinit, float* ws, const Dims& d, Elt t,
                            cudaStream_t s);

// Backward on the tcgen05 tensor cores (bf16, the block decomposition in
// 128-token chunks): the shapes it covers, its workspace, and the launch.
bool backward_tc_supported(const Dims& d, Elt t);
size_t backward_tc_workspace_bytes(const Dims& d);
cudaError_t launch_backward_tc(const void* x, const float* dt, const float* A, const void* B,
                               const void* C, const float* D, const float* init, const void* dy,
                               const float* dfinal, float* dx, float* ddt, float* dA, float* dB,
                               float* dC, float* dD, float* dinit, void* ws, const Dims& d,
                               cudaStream_t s);

}  // namespace ssd
