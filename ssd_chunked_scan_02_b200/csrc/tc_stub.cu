#include "tc_kernels.h"
namespace ssd {
bool tc_supported(const Dims&, Elt) { return false; }
cudaError_t launch_chunk_state_tc(const void*, const float*, const float*, const void*, float*,
                                  float*, const Dims&, cudaStream_t) {
    return cudaErrorNotSupported;
}
cudaError_t launch_chunk_out_tc(const void*, const float*, const float*, const void*, const void*,
                                const float*, const void*, void*, const Dims&, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace ssd
