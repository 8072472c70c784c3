// ssd_noalloc.cu -- ssd_chunk_scan_fwd for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain scratch memory: a plugin loaded into a
// host runtime that owns the whole device heap and hands its plugins no
// allocator, or a latency-critical path where the implicit device-wide
// synchronisation of cudaMalloc/cudaFree is not acceptable.  For them this
// entry point runs the same forward with its scratch taken from a fixed
// array in this library's device memory instead of a caller workspace.
//
// The array is a file-scope __device__ object of SSD_NOALLOC_SCRATCH_BYTES
// bytes.  It is created when the library's device code is loaded on a GPU
// and stays resident on every GPU that loads it until the process exits.
// Host code cannot use the array's name as a device address (on the host it
// names a host-side stand-in), so the device address is looked up with
// cudaGetSymbolAddress once per device, on the first call made while that
// device is current; make that first call before any stream capture begins.
// The address is cached per device ordinal for the life of the process, which
// assumes the device's primary context throughout: no cudaDeviceReset, and no
// other driver-API context made current between calls.
//
// Every call shares the one array and leaves its last contents behind.  The
// forward writes every scratch byte it reads earlier in the same call, so
// nothing needs clearing between calls; but two calls whose work overlaps
// on the GPU (different streams, or different host threads) race on the
// array and must be serialised by the caller.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/ssd.h"

namespace ssd {
void set_error_detail(const char* fmt, ...);
}

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" SSD_API ssd_status_t ssd_chunk_scan_fwd_noalloc(
    const void* x, const float* dt, const float* A, const void* B, const void* C,
    const float* D, int chunk_size, const float* init_states, void* y, float* final_states,
    const ssd_dims_t* dims, ssd_dtype_t dtype, void* stream) {
    // Size check first: it needs no device and rejects oversize problems
    // before anything else happens.
    size_t need = 0;
    ssd_status_t st = ssd_chunk_scan_fwd_workspace_size(dims, chunk_size, dtype, &need);
    if (st != SSD_OK) return st;
    if (need > (size_t)SSD_NOALLOC_SCRATCH_BYTES) {
        ssd::set_error_detail(
            "ssd_chunk_scan_fwd_noalloc: these sizes need %zu bytes of scratch, more than the "
            "%zu bytes built into the library; use ssd_chunk_scan_fwd with a caller workspace",
            need, (size_t)SSD_NOALLOC_SCRATCH_BYTES);
        return SSD_ERR_UNSUPPORTED;
    }

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        ssd::set_error_detail("ssd_chunk_scan_fwd_noalloc: no usable current CUDA device");
        return SSD_ERR_CUDA;
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_ptr[dev]) {
            void* p = nullptr;
            cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess || p == nullptr) {
                ssd::set_error_detail("ssd_chunk_scan_fwd_noalloc: cudaGetSymbolAddress: %s",
                                      cudaGetErrorString(e));
                return SSD_ERR_CUDA;
            }
            g_scratch_ptr[dev] = p;
        }
        scratch = g_scratch_ptr[dev];
    }
    return ssd_chunk_scan_fwd(x, dt, A, B, C, D, chunk_size, init_states, y, final_states, dims,
                              dtype, scratch, (size_t)SSD_NOALLOC_SCRATCH_BYTES, stream);
}
