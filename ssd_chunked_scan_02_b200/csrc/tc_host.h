// tc_host.h -- host helpers shared by the tcgen05 kernel launchers.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"

namespace ssd {

// Encodes a bf16 tiled tensor map with 128-byte swizzle and zero fill for
// out-of-range elements.  dims[0] is the innermost (contiguous) dimension;
// strides_bytes[i] is the byte stride of dims[i + 1].
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box);

// fp32 tiled tensor map: dense row-major boxes in shared memory, or with the
// 128-byte swizzle (box rows of 32 floats, 16-byte chunk c of row r at c ^ (r % 8)).
cudaError_t make_tmap_f32_plain(CUtensorMap* map, const void* base, int rank,
                                const uint64_t* dims, const uint64_t* strides_bytes,
                                const uint32_t* box, bool swizzle128 = false);

bool tma_encoder_available();

// Device address of the status word that bounded waits write (current
// device; looked up once per device ordinal and kept for the process, which
// assumes the device's primary context throughout).  nullptr if unavailable.
unsigned int* device_status_ptr();

// Launches one CTA whose bounded mbarrier wait (at most `polls` polls) is
// bound to give up, recording SSD_ERR_TIMEOUT in the device status word.
cudaError_t launch_expire_wait(uint32_t polls, cudaStream_t s);

// Status word and a fresh token for one launch's bounded waits.
sm100::WaitCtx make_wait_ctx();

// Copies the device status word to the host (synchronising `s`) and clears it.
cudaError_t read_and_clear_device_status(unsigned int* out, cudaStream_t s);

}  // namespace ssd
