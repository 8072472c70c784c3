// tc_host.cu -- host-side support for the tcgen05 kernels: which shapes they
// cover, TMA tensor-map encoding (through the driver entry point, so the
// library does not link libcuda), and the device status word that bounded
// waits write when they give up.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/ssd.h"
#include "sm100.cuh"
#include "tc_host.h"
#include "tc_kernels.h"

namespace ssd {
namespace {
// Device status word: 0 = fine, 4 = a bounded wait in a kernel gave up.
__device__ unsigned int g_device_status = 0;
constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
unsigned int* g_status_ptr[kMaxDevices] = {};
}  // namespace

unsigned int* device_status_ptr() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<unsigned int*>(p);
    }
    return g_status_ptr[dev];
}

sm100::WaitCtx make_wait_ctx() {
    static std::atomic<unsigned int> next{1};
    unsigned int tok = next.fetch_add(1);
    if (tok == 0) tok = next.fetch_add(1);   // 0 means "no timeout"
    return sm100::WaitCtx{device_status_ptr(), tok};
}

bool tc_supported(const Dims& d, Elt t) {
    if (t != Elt::BF16) return false;
    // k virtual heads of headdim 64, or one padded from 32
    if (d.P != 32 && (d.P % 64 != 0 || d.P > 256)) return false;
    if (d.N != 64 && d.N != 128) return false;
    if (d.Q != 128 && d.Q != 256) return false;
    if (d.L <= 0 || d.b <= 0) return false;
    if (d.L > 0x7fffffffLL || d.b > 0x7fffffffLL) return false;   // TMA coordinates are int32
    if (d.H * (d.P / 64) > 0x7fffffffLL / 64) return false;       // head rows of the state maps
    return true;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

bool tma_encoder_available() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box) {
    if (!tma_encoder_available()) return cudaErrorNotSupported;
    cuuint32_t estride[5] = {1, 1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                          const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
                          reinterpret_cast<const cuuint64_t*>(strides_bytes),
                          reinterpret_cast<const cuuint32_t*>(box), estride,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_f32_plain(CUtensorMap* map, const void* base, int rank,
                                const uint64_t* dims, const uint64_t* strides_bytes,
                                const uint32_t* box, bool swizzle128) {
    if (!tma_encoder_available()) return cudaErrorNotSupported;
    cuuint32_t estride[5] = {1, 1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (cuuint32_t)rank,
                          const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
                          reinterpret_cast<const cuuint64_t*>(strides_bytes),
                          reinterpret_cast<const cuuint32_t*>(box), estride,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {
// One thread waits, with at most `polls` polls, on an mbarrier that nothing
// arrives at: the bounded wait gives up and records the timeout status.
__global__ void expire_wait_kernel(uint32_t polls, sm100::WaitCtx status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
    sm100::mbar_wait_polls(&bar, 0, polls, status);
}
}  // namespace

cudaError_t launch_expire_wait(uint32_t polls, cudaStream_t s) {
    const sm100::WaitCtx status = make_wait_ctx();
    if (!status.word) return cudaErrorUnknown;
    expire_wait_kernel<<<1, 32, 0, s>>>(polls, status);
    return cudaGetLastError();
}

cudaError_t read_and_clear_device_status(unsigned int* out, cudaStream_t s) {
    unsigned int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(v), 0,
                                              cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    if (v != 0) {
        e = cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(zero), 0,
                                    cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return e;
        e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return e;
    }
    *out = v;
    return cudaSuccess;
}

}  // namespace ssd
