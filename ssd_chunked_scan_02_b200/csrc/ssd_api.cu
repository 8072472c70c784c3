// ssd_api.cu -- the C ABI declared in include/ssd.h: host-side validation,
// workspace layout, kernel selection and launches.  Nothing here allocates
// device memory or synchronises the device.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include "../../include/ssd.h"
#include "seqpar.h"
#include "ssd_internal.h"
#include "tc_host.h"
#include "tc_kernels.h"

namespace {

thread_local char g_detail[512] = "";

ssd_status_t fail(ssd_status_t s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return s;
}

ssd_status_t cuda_fail(cudaError_t e, const char* where) {
    return fail(SSD_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

size_t elt_size(ssd::Elt t) { return t == ssd::Elt::F32 ? 4 : 2; }

// Validates sizes; fills `out`.  need_chunk: chunk_size is meaningful.
ssd_status_t check_dims(const ssd_dims_t* dims, int chunk, bool need_chunk, ssd_dtype_t dtype,
                        ssd::Dims* out, ssd::Elt* elt) {
    if (!dims) return fail(SSD_ERR_INVALID_ARG, "dims is NULL");
    const ssd_dims_t& d = *dims;
    if (d.batch < 0 || d.seqlen < 0)
        return fail(SSD_ERR_INVALID_ARG, "batch (%lld) and seqlen (%lld) must be >= 0",
                    (long long)d.batch, (long long)d.seqlen);
    if (d.nheads < 1 || d.headdim < 1 || d.dstate < 1 || d.ngroups < 1)
        return fail(SSD_ERR_INVALID_ARG, "nheads, headdim, dstate, ngroups must be >= 1");
    if (d.nheads % d.ngroups != 0)
        return fail(SSD_ERR_INVALID_ARG, "nheads (%lld) must be a multiple of ngroups (%lld)",
                    (long long)d.nheads, (long long)d.ngroups);
    if (d.headdim > 256 || d.dstate > 256)
        return fail(SSD_ERR_UNSUPPORTED, "headdim and dstate must be <= 256");
    if (d.nheads > 65535) return fail(SSD_ERR_UNSUPPORTED, "nheads must be <= 65535");
    if (dtype != SSD_F32 && dtype != SSD_BF16)
        return fail(SSD_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    int Q = 1;
    if (need_chunk) {
        if (chunk < 16 || chunk > 256 || (chunk & (chunk - 1)) != 0)
            return fail(SSD_ERR_UNSUPPORTED, "chunk_size must be a power of two in [16, 256], got %d",
                        chunk);
        Q = chunk;
    }
    const int64_t T = need_chunk ? (d.seqlen + Q - 1) / Q : 1;
    if (d.batch * T > 0x7fffffffLL)
        return fail(SSD_ERR_UNSUPPORTED, "batch * number of chunks exceeds 2^31 - 1");
    out->b = d.batch; out->L = d.seqlen; out->H = d.nheads; out->P = d.headdim;
    out->N = d.dstate; out->G = d.ngroups; out->Q = Q; out->T = T;
    *elt = dtype == SSD_F32 ? ssd::Elt::F32 : ssd::Elt::BF16;
    return SSD_OK;
}

// The fused forward's tensor-core kernels (headdim 32 included), and the
// step entry points' (whose state buffers are the caller's: multiples of 64).
bool fwd_tc(const ssd::Dims& d, ssd::Elt t) { return ssd::tc_supported(d, t); }
bool tc_eligible(const ssd::Dims& d, ssd::Elt t) { return ssd::tc_supported(d, t) && d.P % 64 == 0; }

// The block size the forward runs with.  The decomposition's result does not
// depend on the block size (beyond rounding); the tensor-core kernels take
// 128- and 256-token blocks, so a bf16 forward asked for smaller blocks runs
// with 128-token blocks on them.  The step entry points keep the caller's
// chunk size exactly (their outputs are per chunk).
ssd::Dims forward_dims(const ssd::Dims& d, ssd::Elt t) {
    if (t != ssd::Elt::BF16 || d.Q >= 128) return d;
    ssd::Dims q = d;
    q.Q = 128;
    q.T = (d.L + 127) / 128;
    return fwd_tc(q, t) ? q : d;
}

// The forward's data flow for these sizes (decided from the sizes alone, so
// the workspace size needs no device).
enum class Flow { Simt = 0, ThreeKernel = 1, Walk = 2, Fused = 3 };

Flow pick_flow(const ssd::Dims& d, ssd::Elt t) {
    if (!fwd_tc(d, t)) return Flow::Simt;
    if (!ssd::walk_preferred(d)) return Flow::ThreeKernel;
    return ssd::walk_out_preferred(d) ? Flow::Fused : Flow::Walk;
}

// Whether a data flow covers these sizes (the SIMT kernels cover all).
bool flow_covers(Flow f, const ssd::Dims& d, ssd::Elt t) {
    switch (f) {
        case Flow::Simt: return true;
        case Flow::ThreeKernel:
        case Flow::Walk: return fwd_tc(d, t);
        case Flow::Fused: return fwd_tc(d, t) && ssd::walk_out_supported(d);
    }
    return false;
}

// The forward's sizes and data flow: the library's choice (requested < 0) or
// the requested SSD_FLOW_* (SSD_ERR_UNSUPPORTED if it does not cover them).
// The tensor-core flows run bf16 blocks of 128 tokens or more.
ssd_status_t resolve_flow(ssd::Dims* d, ssd::Elt t, int requested, Flow* f) {
    if (requested < 0) {
        *d = forward_dims(*d, t);
        *f = pick_flow(*d, t);
        return SSD_OK;
    }
    if (requested > (int)Flow::Fused) return fail(SSD_ERR_INVALID_ARG, "unknown data flow %d", requested);
    *f = static_cast<Flow>(requested);
    if (*f != Flow::Simt) *d = forward_dims(*d, t);
    if (!flow_covers(*f, *d, t))
        return fail(SSD_ERR_UNSUPPORTED, "data flow %d does not cover these sizes", requested);
    return SSD_OK;
}

// Workspace regions (each 256-byte aligned).  The three-kernel flows keep the
// chunk states (fp32) and log-decays; the walk keeps its chunk states on chip
// and needs only the entering states.
struct WsLayout {
    size_t states, logdecay, prev, sched, total;
};

WsLayout ws_layout(const ssd::Dims& d, ssd::Elt t, Flow flow) {
    // the tensor-core flows keep 64 state rows for a head of headdim 32
    const int64_t rows = flow == Flow::Simt ? d.P : ssd::state_rows(d.P);
    const size_t nstate = (size_t)(d.b * d.T * d.H) * (size_t)(rows * d.N);
    WsLayout w;
    w.states = 0;
    if (flow == Flow::Walk || flow == Flow::Fused) {
        w.logdecay = 0;
        w.prev = 0;
    } else {
        w.logdecay = round_up(nstate * 4, 256);
        w.prev = w.logdecay + round_up((size_t)(d.b * d.T * d.H) * 4, 256);
    }
    w.sched = w.prev + round_up(nstate * elt_size(t), 256);
    // the fused flow's ticket counter and walker progress flags
    w.total = w.sched + (flow == Flow::Fused ? round_up(ssd::walk_out_sched_bytes(d), 256) : 0);
    if (nstate == 0) w.total = 0;
    return w;
}

// A tensor handed to the kernels must be device memory of the current device:
// tensor maps, the status word and scratch are looked up per current device,
// and a kernel on one GPU given another GPU's (or unregistered host) memory
// faults or reads the wrong memory.  Checked once per call, after every other
// validation, on the call's main input.
ssd_status_t check_current_device(const void* p, const char* name) {
    cudaPointerAttributes a{};
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e, "cudaPointerGetAttributes");
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
        return fail(SSD_ERR_INVALID_ARG, "%s is not device memory", name);
    int dev = -1;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (a.type == cudaMemoryTypeDevice && a.device != dev)
        return fail(SSD_ERR_INVALID_ARG, "%s is on device %d but device %d is current", name,
                    a.device, dev);
    return SSD_OK;
}

#define REQUIRE_DEVICE(p)                                                                \
    do {                                                                                 \
        ssd_status_t st_dev_ = check_current_device((p), #p);                            \
        if (st_dev_ != SSD_OK) return st_dev_;                                           \
    } while (0)

#define REQUIRE_PTR(p)                                                                   \
    do {                                                                                 \
        if (!(p)) return fail(SSD_ERR_INVALID_ARG, "%s is NULL", #p);                    \
        if (!aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
    } while (0)
#define OPTIONAL_PTR(p)                                                                  \
    do {                                                                                 \
        if ((p) && !aligned16(p))                                                        \
            return fail(SSD_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p);           \
    } while (0)

}  // namespace

namespace ssd {
// Records a message for ssd_last_error_detail() on this host thread.
void set_error_detail(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
}
}  // namespace ssd

extern "C" {

const char* ssd_status_string(ssd_status_t s) {
    switch (s) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA";
        case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT";
    }
    return "SSD_ERR_UNKNOWN";
}

const char* ssd_last_error_detail(void) { return g_detail; }

ssd_status_t ssd_chunk_scan_fwd_flow_workspace_size(const ssd_dims_t* dims, int chunk_size,
                                                    ssd_dtype_t dtype, int flow, size_t* bytes) {
    g_detail[0] = 0;
    if (!bytes) return fail(SSD_ERR_INVALID_ARG, "bytes is NULL");
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, chunk_size, true, dtype, &d, &t);
    if (st != SSD_OK) return st;
    Flow f = Flow::Simt;
    st = resolve_flow(&d, t, flow, &f);
    if (st != SSD_OK) return st;
    *bytes = ws_layout(d, t, f).total;
    return SSD_OK;
}

ssd_status_t ssd_chunk_scan_fwd_workspace_size(const ssd_dims_t* dims, int chunk_size,
                                               ssd_dtype_t dtype, size_t* bytes) {
    return ssd_chunk_scan_fwd_flow_workspace_size(dims, chunk_size, dtype, -1, bytes);
}

int ssd_chunk_scan_fwd_uses_tensor_cores(const ssd_dims_t* dims, int chunk_size,
                                         ssd_dtype_t dtype) {
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    if (check_dims(dims, chunk_size, true, dtype, &d, &t) != SSD_OK) return -1;
    return fwd_tc(forward_dims(d, t), t) ? 1 : 0;
}

int ssd_chunk_scan_fwd_data_flow(const ssd_dims_t* dims, int chunk_size, ssd_dtype_t dtype) {
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    if (check_dims(dims, chunk_size, true, dtype, &d, &t) != SSD_OK) return -1;
    switch (pick_flow(forward_dims(d, t), t)) {
        case Flow::Fused: return SSD_FLOW_WALK_OUTPUT_FUSED;
        case Flow::Walk: return SSD_FLOW_WALK_OUTPUT;
        case Flow::ThreeKernel: return SSD_FLOW_TC_THREE_KERNEL;
        default: return SSD_FLOW_SIMT;
    }
}

ssd_status_t ssd_chunk_scan_fwd(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, int chunk_size,
                                const float* init_states, void* y, float* final_states,
                                const ssd_dims_t* dims, ssd_dtype_t dtype, void* workspace,
                                size_t workspace_bytes, void* stream) {
    return ssd_chunk_scan_fwd_with_flow(x, dt, A, B, C, D, chunk_size, init_states, y,
                                        final_states, dims, dtype, workspace, workspace_bytes,
                                        stream, -1);
}

ssd_status_t ssd_chunk_scan_fwd_with_flow(const void* x, const float* dt, const float* A,
                                          const void* B, const void* C, const float* D,
                                          int chunk_size, const float* init_states, void* y,
                                          float* final_states, const ssd_dims_t* dims,
                                          ssd_dtype_t dtype, void* workspace,
                                          size_t workspace_bytes, void* stream, int flow_req) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, chunk_size, true, dtype, &d, &t);
    if (st != SSD_OK) return st;
    Flow flow = Flow::Simt;
    st = resolve_flow(&d, t, flow_req, &flow);
    if (st != SSD_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    OPTIONAL_PTR(init_states);
    OPTIONAL_PTR(final_states);
    if (d.b == 0) return SSD_OK;
    if (d.L == 0) {
        if (!final_states) return SSD_OK;
        cudaError_t e = ssd::launch_copy_or_zero(init_states, final_states, d.b * d.H * d.P * d.N, s);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "final-state copy");
    }
    REQUIRE_PTR(x); REQUIRE_PTR(dt); REQUIRE_PTR(A); REQUIRE_PTR(B); REQUIRE_PTR(C);
    REQUIRE_PTR(D); REQUIRE_PTR(y);
    const WsLayout w = ws_layout(d, t, flow);
    if (workspace_bytes < w.total)
        return fail(SSD_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed",
                    workspace_bytes, w.total);
    REQUIRE_PTR(workspace);
    if (!aligned16(workspace)) return fail(SSD_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    REQUIRE_DEVICE(x);
    char* ws = static_cast<char*>(workspace);
    float* states = reinterpret_cast<float*>(ws + w.states);
    float* logdecay = reinterpret_cast<float*>(ws + w.logdecay);
    void* prev = ws + w.prev;

    cudaError_t e;
    if (flow == Flow::Fused) {
        e = ssd::launch_walk_out_tc(x, dt, A, B, C, D, init_states, prev, y, final_states,
                                    reinterpret_cast<int*>(ws + w.sched), d, s);
        if (e != cudaSuccess) return cuda_fail(e, "walk + output kernel (tcgen05)");
        return SSD_OK;
    }
    if (flow == Flow::Walk) {
        e = ssd::launch_state_walk_tc(x, dt, A, B, init_states, prev, final_states, d, s);
        if (e != cudaSuccess) return cuda_fail(e, "state-walk kernel (tcgen05)");
        e = ssd::launch_chunk_out_tc(x, dt, A, B, C, D, prev, y, d, s);
        if (e != cudaSuccess) return cuda_fail(e, "chunk-output kernel (tcgen05)");
        return SSD_OK;
    }
    if (flow == Flow::ThreeKernel) {
        e = ssd::launch_chunk_state_tc(x, dt, A, B, states, logdecay, d, s);
        if (e != cudaSuccess) return cuda_fail(e, "chunk-state kernel (tcgen05)");
        // the state buffers have state_rows(P) rows a head; init and final P
        ssd::Dims ds = d;
        ds.P = ssd::state_rows(d.P);
        e = ssd::launch_state_pass(states, logdecay, init_states, prev, final_states, ds, t, s,
                                   false, d.P);
        if (e != cudaSuccess) return cuda_fail(e, "state-passing kernel");
        e = ssd::launch_chunk_out_tc(x, dt, A, B, C, D, prev, y, d, s);
        if (e != cudaSuccess) return cuda_fail(e, "chunk-output kernel (tcgen05)");
        return SSD_OK;
    }
    e = ssd::launch_chunk_state_simt(x, dt, A, B, states, logdecay, d, t, s);
    if (e != cudaSuccess) return cuda_fail(e, "chunk-state kernel");
    e = ssd::launch_state_pass(states, logdecay, init_states, prev, final_states, d, t, s);
    if (e != cudaSuccess) return cuda_fail(e, "state-passing kernel");
    e = ssd::launch_chunk_out_simt(x, dt, A, B, C, D, prev, y, d, t, s);
    if (e != cudaSuccess) return cuda_fail(e, "chunk-output kernel");
    return SSD_OK;
}

ssd_status_t ssd_chunk_state_fwd(const void* x, const float* dt, const float* A, const void* B,
                                 int chunk_size, float* chunk_states, float* chunk_logdecay,
                                 const ssd_dims_t* dims, ssd_dtype_t dtype, void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, chunk_size, true, dtype, &d, &t);
    if (st != SSD_OK) return st;
    if (d.b == 0 || d.L == 0) return SSD_OK;
    REQUIRE_PTR(x); REQUIRE_PTR(dt); REQUIRE_PTR(A); REQUIRE_PTR(B);
    REQUIRE_PTR(chunk_states); REQUIRE_PTR(chunk_logdecay);
    REQUIRE_DEVICE(x);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = tc_eligible(d, t)
                        ? ssd::launch_chunk_state_tc(x, dt, A, B, chunk_states, chunk_logdecay, d, s)
                        : ssd::launch_chunk_state_simt(x, dt, A, B, chunk_states, chunk_logdecay,
                                                       d, t, s);
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "chunk-state kernel");
}

ssd_status_t ssd_state_passing_fwd(const float* chunk_states, const float* chunk_logdecay,
                                   const float* init_states, void* prev_states,
                                   float* final_states, int chunk_size, const ssd_dims_t* dims,
                                   ssd_dtype_t dtype, void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, chunk_size, true, dtype, &d, &t);
    if (st != SSD_OK) return st;
    OPTIONAL_PTR(init_states);
    OPTIONAL_PTR(final_states);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d.b == 0) return SSD_OK;
    if (d.L == 0) {
        if (!final_states) return SSD_OK;
        cudaError_t e = ssd::launch_copy_or_zero(init_states, final_states, d.b * d.H * d.P * d.N, s);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "final-state copy");
    }
    REQUIRE_PTR(chunk_states); REQUIRE_PTR(chunk_logdecay); REQUIRE_PTR(prev_states);
    REQUIRE_DEVICE(chunk_states);
    cudaError_t e = ssd::launch_state_pass(chunk_states, chunk_logdecay, init_states, prev_states,
                                           final_states, d, t, s);
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "state-passing kernel");
}

ssd_status_t ssd_chunk_output_fwd(const void* x, const float* dt, const float* A, const void* B,
                                  const void* C, const float* D, const void* prev_states,
                                  int chunk_size, void* y, const ssd_dims_t* dims,
                                  ssd_dtype_t dtype, void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, chunk_size, true, dtype, &d, &t);
    if (st != SSD_OK) return st;
    if (d.b == 0 || d.L == 0) return SSD_OK;
    REQUIRE_PTR(x); REQUIRE_PTR(dt); REQUIRE_PTR(A); REQUIRE_PTR(B); REQUIRE_PTR(C);
    REQUIRE_PTR(D); REQUIRE_PTR(prev_states); REQUIRE_PTR(y);
    REQUIRE_DEVICE(x);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = tc_eligible(d, t)
                        ? ssd::launch_chunk_out_tc(x, dt, A, B, C, D, prev_states, y, d, s)
                        : ssd::launch_chunk_out_simt(x, dt, A, B, C, D, prev_states, y, d, t, s);
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "chunk-output kernel");
}

ssd_status_t ssd_state_walk_fwd(const void* x, const float* dt, const float* A, const void* B,
                                const float* init_states, void* prev_states, float* final_states,
                                int chunk_size, const ssd_dims_t* dims, ssd_dtype_t dtype,
                                void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, chunk_size, true, dtype, &d, &t);
    if (st != SSD_OK) return st;
    OPTIONAL_PTR(init_states);
    OPTIONAL_PTR(final_states);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d.b == 0) return SSD_OK;
    if (d.L == 0) {
        if (!final_states) return SSD_OK;
        cudaError_t e = ssd::launch_copy_or_zero(init_states, final_states, d.b * d.H * d.P * d.N, s);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "final-state copy");
    }
    if (!tc_eligible(d, t))
        return fail(SSD_ERR_UNSUPPORTED,
                    "the state walk covers bf16, chunk 128/256, headdim 64/128/192/256 and "
                    "dstate 64/128");
    REQUIRE_PTR(x); REQUIRE_PTR(dt); REQUIRE_PTR(A); REQUIRE_PTR(B); REQUIRE_PTR(prev_states);
    REQUIRE_DEVICE(x);
    cudaError_t e = ssd::launch_state_walk_tc(x, dt, A, B, init_states, prev_states, final_states, d, s);
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "state-walk kernel");
}

// ---------------------------------------------------------------- sequence parallelism
ssd_status_t ssd_seq_logdecay(const float* dt, const float* A, float* logdecay,
                              const ssd_dims_t* dims, void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, 0, false, SSD_F32, &d, &t);
    if (st != SSD_OK) return st;
    if (d.b == 0) return SSD_OK;
    REQUIRE_PTR(A); REQUIRE_PTR(logdecay);
    if (d.L > 0) REQUIRE_PTR(dt);
    REQUIRE_DEVICE(logdecay);
    cudaError_t e = ssd::launch_seq_logdecay(dt, A, logdecay, d, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "log-decay kernel");
}

ssd_status_t ssd_state_exchange_combine(const float* local_final, const float* logdecay,
                                        const float* init, int rank, int nranks, float* h_in,
                                        const ssd_dims_t* dims, void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, 0, false, SSD_F32, &d, &t);
    if (st != SSD_OK) return st;
    if (nranks < 1 || rank < 0 || rank > nranks)
        return fail(SSD_ERR_INVALID_ARG, "need 0 <= rank (%d) <= nranks (%d), nranks >= 1", rank,
                    nranks);
    OPTIONAL_PTR(init);
    if (d.b == 0) return SSD_OK;
    REQUIRE_PTR(h_in);
    if (rank > 0) {
        REQUIRE_PTR(local_final);
        REQUIRE_PTR(logdecay);
    }
    REQUIRE_DEVICE(h_in);
    cudaError_t e = ssd::launch_state_combine(local_final, logdecay, init, h_in, rank, d,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "state-combine kernel");
}

namespace {
struct CorrLayout {
    size_t prefix, hbf, total;
};
CorrLayout corr_layout(const ssd::Dims& d, ssd::Elt t) {
    CorrLayout c;
    c.prefix = 0;
    c.hbf = round_up((size_t)(d.b * ssd::correction_tiles(d) * d.H) * 4, 256);
    c.total = c.hbf;
    if (ssd::correction_tc_supported(d, t)) c.total += round_up((size_t)(d.b * d.H * d.P * d.N) * 2, 256);
    if (d.b == 0 || d.L == 0) c.total = 0;
    return c;
}
}  // namespace

ssd_status_t ssd_state_correction_workspace_size(const ssd_dims_t* dims, ssd_dtype_t dtype,
                                                 size_t* bytes) {
    g_detail[0] = 0;
    if (!bytes) return fail(SSD_ERR_INVALID_ARG, "bytes is NULL");
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, 0, false, dtype, &d, &t);
    if (st != SSD_OK) return st;
    *bytes = corr_layout(d, t).total;
    return SSD_OK;
}

ssd_status_t ssd_state_correction_fwd(const float* h_in, const float* dt, const float* A,
                                      const void* C, void* y, float* final_states,
                                      const ssd_dims_t* dims, ssd_dtype_t dtype,
                                      void* workspace, size_t workspace_bytes, void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, 0, false, dtype, &d, &t);
    if (st != SSD_OK) return st;
    OPTIONAL_PTR(final_states);
    if (d.b == 0 || d.L == 0) return SSD_OK;     // an empty shard: h_in passes through unchanged
    REQUIRE_PTR(h_in); REQUIRE_PTR(dt); REQUIRE_PTR(A); REQUIRE_PTR(C); REQUIRE_PTR(y);
    const CorrLayout w = corr_layout(d, t);
    if (workspace_bytes < w.total)
        return fail(SSD_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed",
                    workspace_bytes, w.total);
    REQUIRE_PTR(workspace);
    REQUIRE_DEVICE(y);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    float* prefix = reinterpret_cast<float*>(ws + w.prefix);
    const bool tc = ssd::correction_tc_supported(d, t);
    __nv_bfloat16* hbf = tc ? reinterpret_cast<__nv_bfloat16*>(ws + w.hbf) : nullptr;
    cudaError_t e = ssd::launch_correction_prep(h_in, dt, A, prefix, final_states, hbf, d, s);
    if (e != cudaSuccess) return cuda_fail(e, "correction prep kernel");
    e = tc ? ssd::launch_correction_tc(hbf, dt, A, C, prefix, y, d, s)
           : ssd::launch_correction_simt(h_in, dt, A, C, prefix, y, d, t, s);
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, tc ? "correction kernel (tcgen05)"
                                                       : "correction kernel");
}

ssd_status_t ssd_debug_expire_wait(unsigned int polls, void* stream) {
    g_detail[0] = 0;
    if (polls < 1 || polls > (1u << 20))
        return fail(SSD_ERR_INVALID_ARG, "polls must be in [1, 2^20], got %u", polls);
    cudaError_t e = ssd::launch_expire_wait(polls, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "expire-wait kernel");
}

ssd_status_t ssd_poll_device_status(void* stream) {
    g_detail[0] = 0;
    unsigned int v = 0;
    cudaError_t e = ssd::read_and_clear_device_status(&v, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "device status read");
    if (v != 0) return fail(SSD_ERR_TIMEOUT, "a bounded device-side wait gave up (code %u)", v);
    return SSD_OK;
}

ssd_status_t ssd_step(float* state, const void* x, const float* dt, const float* A,
                      const void* B, const void* C, const float* D, void* y,
                      const ssd_dims_t* dims, ssd_dtype_t dtype, void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, 0, false, dtype, &d, &t);
    if (st != SSD_OK) return st;
    if (d.b == 0) return SSD_OK;
    REQUIRE_PTR(state); REQUIRE_PTR(x); REQUIRE_PTR(dt); REQUIRE_PTR(A); REQUIRE_PTR(B);
    REQUIRE_PTR(C); REQUIRE_PTR(D); REQUIRE_PTR(y);
    REQUIRE_DEVICE(state);
    cudaError_t e = ssd::launch_step(state, x, dt, A, B, C, D, y, d, t,
                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "decode-step kernel");
}

ssd_status_t ssd_chunk_scan_bwd_workspace_size(const ssd_dims_t* dims, ssd_dtype_t dtype,
                                               size_t* bytes) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, 0, false, dtype, &d, &t);
    if (st != SSD_OK) return st;
    if (!bytes) return fail(SSD_ERR_INVALID_ARG, "bytes is NULL");
    if (d.b == 0 || d.L == 0) {
        *bytes = 0;
        return SSD_OK;
    }
    if (ssd::backward_tc_supported(d, t)) {
        *bytes = ssd::backward_tc_workspace_bytes(d);
        return SSD_OK;
    }
    if (!ssd::backward_supported(d))
        return fail(SSD_ERR_UNSUPPORTED, "dstate too large for the backward");
    *bytes = ssd::backward_workspace_bytes(d);
    return SSD_OK;
}

int ssd_chunk_scan_bwd_uses_tensor_cores(const ssd_dims_t* dims, ssd_dtype_t dtype) {
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    if (check_dims(dims, 0, false, dtype, &d, &t) != SSD_OK) return -1;
    if (ssd::backward_tc_supported(d, t)) return 1;
    return ssd::backward_supported(d) ? 0 : -1;
}

ssd_status_t ssd_chunk_scan_bwd(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, const float* init_states,
                                const void* dy, const float* dfinal_states, float* dx,
                                float* ddt, float* dA, float* dB, float* dC, float* dD,
                                float* dinit_states, const ssd_dims_t* dims, ssd_dtype_t dtype,
                                void* workspace, size_t workspace_bytes, void* stream) {
    g_detail[0] = 0;
    ssd::Dims d{}; ssd::Elt t = ssd::Elt::BF16;
    ssd_status_t st = check_dims(dims, 0, false, dtype, &d, &t);
    if (st != SSD_OK) return st;
    const bool tc = d.b > 0 && d.L > 0 && ssd::backward_tc_supported(d, t);
    if (!tc && !ssd::backward_supported(d))
        return fail(SSD_ERR_UNSUPPORTED, "dstate too large for the backward");
    REQUIRE_PTR(A); REQUIRE_PTR(D); REQUIRE_PTR(dA); REQUIRE_PTR(dD);
    OPTIONAL_PTR(init_states); OPTIONAL_PTR(dfinal_states); OPTIONAL_PTR(dinit_states);
    if (d.b > 0 && d.L > 0) {
        REQUIRE_PTR(x); REQUIRE_PTR(dt); REQUIRE_PTR(B); REQUIRE_PTR(C); REQUIRE_PTR(dy);
        REQUIRE_PTR(dx); REQUIRE_PTR(ddt); REQUIRE_PTR(dB); REQUIRE_PTR(dC);
        const size_t need = tc ? ssd::backward_tc_workspace_bytes(d) : ssd::backward_workspace_bytes(d);
        if (workspace_bytes < need)
            return fail(SSD_ERR_INVALID_ARG, "workspace_bytes %zu < required %zu", workspace_bytes,
                        need);
        REQUIRE_PTR(workspace);
        REQUIRE_DEVICE(x);
    }
    if (tc) {
        cudaError_t e = ssd::launch_backward_tc(x, dt, A, B, C, D, init_states, dy, dfinal_states,
                                                dx, ddt, dA, dB, dC, dD, dinit_states, workspace,
                                                d, static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "backward kernels (tcgen05)");
    }
    cudaError_t e = ssd::launch_backward(x, dt, A, B, C, D, init_states, dy, dfinal_states, dx,
                                         ddt, dA, dB, dC, dD, dinit_states,
                                         static_cast<float*>(workspace), d, t,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "backward kernel");
}

}  // extern "C"
