/*
 * ssd.h -- C ABI of libssd_b200.so, a B200 (sm_100a) implementation of the
 * SSD (structured state space duality) layer of Mamba-2.
 *
 * The layer (scalar-times-identity A per head, input-dependent dt, B, C):
 *
 *     h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T        (P x N state per head)
 *     y_t = h_t C_t + D_h * x_t
 *
 * "论文解读：Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
 * section 状态空间模型: discretise (Delta, A, B) and run the model as a linear
 * recurrence; section 选择性状态空间模型: dt, B, C vary per token.
 * "Transformers are SSMs" (CiteArk), AI research summary: the same map is a
 * 1-semiseparable matrix, evaluated by a block-decomposed matrix-multiply
 * algorithm on the tensor cores; "what this means": the recurrent form gives
 * constant-memory inference (ssd_step below).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer (cudaMalloc'd or equivalent),
 *    dense, row-major and contiguous, and 16-byte aligned.  The caller owns
 *    all memory, including the workspace; the library never allocates.
 *  - Layouts (b = batch, L = seqlen, H = nheads, P = headdim, N = dstate,
 *    G = ngroups, T = ceil(L / chunk_size)):
 *        x, y            (b, L, H, P)   element type = dtype
 *        dt              (b, L, H)      fp32, already positive (no softplus is applied)
 *        A, D            (H)            fp32 (A <= 0: a decaying state, see below)
 *        B, C            (b, L, G, N)   element type = dtype
 *        states          (b, H, P, N)   fp32 (init_states, final_states, ssd_step's state)
 *    Head h reads B/C group g = h / (H / G).
 *  - dtype: SSD_F32 (all fp32; exact fp32 arithmetic) or SSD_BF16 (x, B, C, y
 *    in bf16; products on the tensor cores with fp32 accumulation; decays,
 *    prefix sums, the inter-chunk recurrence and all states in fp32).
 *  - A: the model's regime is A <= 0 (exp(dt*A) <= 1); the tensor-core
 *    kernels factorise the decay through per-row and per-column factors that
 *    are exact for any A <= 0.  A > 0 (a growing state) is computed
 *    correctly as long as the growth over one chunk, exp(sum dt*A), stays
 *    below 2^60; beyond that the result overflows fp32 in any case.
 *  - Sizes are passed as a pointer to ssd_dims_t (a by-value struct of six
 *    int64 is awkward for some FFI layers; the pointee is only read, during
 *    the call), and the stream as void* (a cudaStream_t, so that this header
 *    does not need the CUDA headers).
 *  - Device: every pointer must belong to the CUDA device that is current
 *    on the calling thread; the library looks up per-device state (tensor
 *    maps, status word, built-in scratch) for that device and assumes its
 *    primary context (do not call cudaDeviceReset between calls).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and runs asynchronously: no call synchronises the device.
 *  - Errors: arguments are validated on the host before anything is
 *    launched; a rejected call launches nothing and writes nothing.  A
 *    failed launch returns SSD_ERR_CUDA (the CUDA error text is available
 *    from ssd_last_error_detail()).  Asynchronous device errors surface at
 *    the caller's next synchronisation, as with any CUDA library.
 *  - Thread safety: calls may be made from several host threads on
 *    different streams; calls that share a workspace must not overlap.
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, too-small workspace */
    SSD_ERR_UNSUPPORTED = 2,  /* well-formed but outside what the kernels implement */
    SSD_ERR_CUDA = 3,         /* a CUDA runtime/driver call or a launch failed */
    SSD_ERR_TIMEOUT = 4       /* a bounded device-side wait gave up (ssd_poll_device_status) */
} ssd_status_t;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype_t;

typedef struct {
    int64_t batch;    /* b >= 0 */
    int64_t seqlen;   /* L >= 0 (any value; a last partial chunk is handled) */
    int64_t nheads;   /* H >= 1 */
    int64_t headdim;  /* P, 1..256 */
    int64_t dstate;   /* N, 1..256 */
    int64_t ngroups;  /* G >= 1, H % G == 0 */
} ssd_dims_t;

/* Human-readable name of a status code (static storage). */
SSD_API const char* ssd_status_string(ssd_status_t s);

/* Detail of the last error raised on the calling host thread (validation
 * message or CUDA error text); "" if none.  Thread-local static storage. */
SSD_API const char* ssd_last_error_detail(void);

/*
 * Bytes of device workspace ssd_chunk_scan_fwd needs for these sizes
 * (chunk states, per-chunk log-decays and the states entering each chunk,
 * as the data flow needs them, and for the one-launch flow a few scheduling
 * counters).
 * Writes the size to *bytes.  Returns SSD_ERR_INVALID_ARG / UNSUPPORTED on
 * sizes that ssd_chunk_scan_fwd would reject.
 */
SSD_API ssd_status_t ssd_chunk_scan_fwd_workspace_size(const ssd_dims_t* dims, int chunk_size,
                                               ssd_dtype_t dtype, size_t* bytes);

/*
 * Chunked (block-decomposed) SSD forward over whole sequences.
 * "Transformers are SSMs" (CiteArk), AI research summary: block-decomposed
 * matrix multiplication of the 1-semiseparable matrix; review page
 * "Review: Transformers are SSMs (Mamba-2)", 核心概念 item 5 (SSD algorithm:
 * block decomposition that uses the tensor cores and stays linear in L).
 * The sequence is cut into chunks of `chunk_size` tokens (a power of two,
 * 16..256; the last chunk may be partial).  The result does not depend on
 * the chunk size beyond rounding; for bf16 the tensor-core kernels run
 * 128- or 256-token chunks, and a smaller chunk_size runs as 128-token
 * chunks on them (the workspace size accounts for it).  Four steps:
 *   (1) per chunk, the intra-chunk quadratic term (C B^T masked by the
 *       exp(segsum(dt*A)) decay) applied to dt*x;
 *   (2) per chunk, the state it contributes, B^T (decay * dt * x);
 *   (3) the sequential recurrence of states across chunks (fp32);
 *   (4) the contribution of the entering state, C * h, plus D_h * x.
 * init_states: (b,H,P,N) fp32, or NULL for zero initial states.
 * final_states: (b,H,P,N) fp32 output, or NULL when not wanted.
 * y: (b,L,H,P) output in dtype.  workspace: >= the size reported by
 * ssd_chunk_scan_fwd_workspace_size (may be NULL only when that size is 0).
 * Inputs and outputs must not alias.
 */
SSD_API ssd_status_t ssd_chunk_scan_fwd(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, int chunk_size,
                                const float* init_states, void* y, float* final_states,
                                const ssd_dims_t* dims, ssd_dtype_t dtype, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * One decode step for a batch of sequences (the recurrent, constant-memory
 * form: "Transformers are SSMs" (CiteArk), "what this means"; Mamba digest,
 * 状态空间模型: the linear-recurrence mode suited to autoregressive inference).
 *   state (b,H,P,N) fp32, updated in place:  state <- exp(dt*A_h) state + dt x B^T
 *   y (b,H,P) in dtype:                      y = state C + D_h x
 * x (b,H,P) dtype; dt (b,H) fp32; B, C (b,G,N) dtype; A, D (H) fp32.
 * dims->seqlen is ignored.
 */
SSD_API ssd_status_t ssd_step(float* state, const void* x, const float* dt, const float* A,
                      const void* B, const void* C, const float* D, void* y,
                      const ssd_dims_t* dims, ssd_dtype_t dtype, void* stream);

/*
 * The forward's steps one at a time (the same kernels ssd_chunk_scan_fwd
 * launches), for testing each step on its own.  T = ceil(L / chunk_size).
 *
 * ssd_chunk_state_fwd -- step (2): chunk_states (b,T,H,P,N) fp32 receives, for
 *   every chunk, the state reached at the chunk's last token when the state
 *   at the chunk's start is zero; chunk_logdecay (b,T,H) fp32 receives
 *   sum_{t in chunk} dt_t * A_h.
 * ssd_state_passing_fwd -- step (3): prev_states (b,T,H,P,N) in dtype
 *   receives the state entering each chunk (h before the chunk's first
 *   token), computed in fp32 as h_c = exp(logdecay_c) h_{c-1} + S_c from
 *   init_states (NULL = zero); final_states (nullable) receives the state
 *   after the last chunk.
 * ssd_chunk_output_fwd -- steps (1) and (4): y from x, dt, A, B, C, D and
 *   prev_states (as written by ssd_state_passing_fwd).
 */
SSD_API ssd_status_t ssd_chunk_state_fwd(const void* x, const float* dt, const float* A, const void* B,
                                 int chunk_size, float* chunk_states, float* chunk_logdecay,
                                 const ssd_dims_t* dims, ssd_dtype_t dtype, void* stream);
SSD_API ssd_status_t ssd_state_passing_fwd(const float* chunk_states, const float* chunk_logdecay,
                                   const float* init_states, void* prev_states,
                                   float* final_states, int chunk_size, const ssd_dims_t* dims,
                                   ssd_dtype_t dtype, void* stream);
SSD_API ssd_status_t ssd_chunk_output_fwd(const void* x, const float* dt, const float* A, const void* B,
                                  const void* C, const float* D, const void* prev_states,
                                  int chunk_size, void* y, const ssd_dims_t* dims,
                                  ssd_dtype_t dtype, void* stream);

/*
 * ssd_chunk_scan_fwd for callers that cannot allocate device memory (a plugin
 * inside a host runtime that owns the device heap and offers no allocator,
 * or a latency-critical path that cannot afford the device-wide
 * synchronisation of cudaMalloc/cudaFree).  The pages describe no
 * counterpart: this is a library convenience, not part of the method.
 * Same arguments and result as ssd_chunk_scan_fwd, without the workspace:
 * the scratch comes from one fixed device array of SSD_NOALLOC_SCRATCH_BYTES
 * inside the library, resident on every GPU that loads the library until
 * the process exits.  Sizes whose workspace (ssd_chunk_scan_fwd_workspace_size)
 * exceeds that return SSD_ERR_UNSUPPORTED with a message.  The first call
 * on each device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current; make it before any stream capture.  The address
 * is kept for the life of the process, per device ordinal: it assumes the
 * device's primary context throughout (no cudaDeviceReset, no other driver
 * context made current between calls).  Nothing is
 * allocated or freed.  All calls share the array and it keeps the last
 * call's contents (every byte read is rewritten first within a call, so no
 * clearing is needed), so calls that overlap on the GPU race: serialise them.
 */
#define SSD_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
SSD_API ssd_status_t ssd_chunk_scan_fwd_noalloc(const void* x, const float* dt, const float* A,
                                                const void* B, const void* C, const float* D,
                                                int chunk_size, const float* init_states,
                                                void* y, float* final_states,
                                                const ssd_dims_t* dims, ssd_dtype_t dtype,
                                                void* stream);

/*
 * Gradients of ssd_chunk_scan_fwd.  "Transformers are SSMs" (CiteArk), AI
 * research summary: training is what the layer is for; the gradients are the
 * chain rule on the recurrence h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T,
 * y_t = h_t C_t + D_h x_t.  Two implementations, chosen from the sizes and
 * dtype (ssd_chunk_scan_bwd_uses_tensor_cores tells which):
 *   - SSD_BF16 with headdim 32 or 64..256 (a multiple of 64) and dstate 64
 *     or 128:
 *     the block decomposition in 128-token chunks on the tcgen05 tensor cores
 *     (the forward's entering states recomputed, a reverse pass over the
 *     chunks for dL/dh, then per chunk the masked products C B^T o E and
 *     dy x^T o E and the state terms), bf16 operands with fp32 accumulation;
 *     the decay gradients come from fp32 products, and the states enter
 *     them as bf16 value + residue pairs (their sums cancel there).
 *     Accuracy: the bf16 bound, 5e-3 of each gradient's largest element.
 *   - everything else (all of SSD_F32): exact fp32 on the CUDA cores, one CTA
 *     per block of state rows of a (batch, head) walking the sequence in
 *     reverse token order (slow next to the forward).
 * Inputs: the forward's inputs (x, B, C in dtype; dt, A, D, init_states
 * fp32; init_states NULL = zero), dy (b,L,H,P) in dtype = dL/dy, and
 * dfinal_states (b,H,P,N) fp32 = dL/dfinal_states or NULL (zero).
 * Outputs, all fp32 and fully written: dx (b,L,H,P), ddt (b,L,H), dA (H),
 * dB (b,L,G,N), dC (b,L,G,N) (summed over the heads of each group), dD (H),
 * dinit_states (b,H,P,N) = dL/dinit_states (NULL = not wanted).  dA and dD
 * (and on the CUDA-core path dB and dC) are zeroed, then accumulated with
 * atomics, so their rounding (not their value) may differ between runs.
 * workspace: >= the size reported by ssd_chunk_scan_bwd_workspace_size
 * (tensor cores: the entering states and dL/dh per 128-token chunk, each
 * as a bf16 value and its bf16 rounding residue, plus one fp32 buffer,
 * b*ceil(L/128)*H*max(P,64)*N*12 bytes and change; CUDA cores:
 * fp32 state checkpoints every 64 tokens and one 64-token segment of
 * states, per (batch, head) and block of state rows); NULL only when that
 * size is 0.  Inputs and outputs must not alias.
 */
SSD_API ssd_status_t ssd_chunk_scan_bwd_workspace_size(const ssd_dims_t* dims, ssd_dtype_t dtype,
                                                       size_t* bytes);
/* Which implementation ssd_chunk_scan_bwd uses for these sizes: 1 = tcgen05
 * tensor cores, 0 = exact fp32 on the CUDA cores, -1 = rejected. */
SSD_API int ssd_chunk_scan_bwd_uses_tensor_cores(const ssd_dims_t* dims, ssd_dtype_t dtype);
SSD_API ssd_status_t ssd_chunk_scan_bwd(const void* x, const float* dt, const float* A,
                                        const void* B, const void* C, const float* D,
                                        const float* init_states, const void* dy,
                                        const float* dfinal_states, float* dx, float* ddt,
                                        float* dA, float* dB, float* dC, float* dD,
                                        float* dinit_states, const ssd_dims_t* dims,
                                        ssd_dtype_t dtype, void* workspace,
                                        size_t workspace_bytes, void* stream);

/*
 * Sequence parallelism: splitting L across ranks with one exchange.
 * "Transformers are SSMs" (CiteArk), what this means: the layer lends
 * itself to large-scale training with model parallelism.  The state is the
 * only thing a later part of the sequence needs from an earlier one, and it
 * enters linearly: with h_in the state entering a shard,
 *     y_t = y_t|zero start + exp(cs_t) h_in C_t,    cs_t = sum_{k <= t} dt_k A_h,
 *     h_end = h_end|zero start + exp(cs_last) h_in
 * (cs from the shard's first token).  So rank r runs ssd_chunk_scan_fwd on
 * its shard from a zero state, takes ssd_seq_logdecay of its shard, and the
 * ranks all-gather (local final state, log-decay) -- b*H*(P*N+1) fp32 per
 * rank; ssd_state_exchange_combine then gives each rank its h_in (the
 * exclusive scan over the ranks before it), and ssd_state_correction_fwd
 * adds h_in's contribution to the shard's y and final state.
 *
 * ssd_seq_logdecay: logdecay (b,H) fp32 = sum over the L tokens of dt[b,t,h]
 *   * A[h] (natural-log units, summed in fp64).  dims->seqlen = the shard's L.
 * ssd_state_exchange_combine: local_final (R,b,H,P,N) fp32 and logdecay
 *   (R,b,H) fp32 are the gathered values of ranks 0..R-1 (rank order);
 *   init (b,H,P,N) fp32 or NULL (zero) is the state entering rank 0's shard.
 *   Writes h_in (b,H,P,N) fp32 = the state entering rank `rank`'s shard:
 *   h_0 = init, h_{q+1} = exp(logdecay_q) h_q + local_final_q, for
 *   0 <= rank <= R (rank = R gives the state after the whole sequence).
 *   dims->seqlen is ignored.
 * ssd_state_correction_fwd: y (b,L,H,P) in dtype is updated in place,
 *   y_t += exp(cs_t) h_in C_t (computed in fp32, rounded once to dtype);
 *   final_states (b,H,P,N) fp32, if non-NULL, is updated in place,
 *   final += exp(cs_last) h_in.  h_in (b,H,P,N) fp32; dt, A, C as in the
 *   forward.  For bf16 with headdim 64..256 (a multiple of 64) and dstate
 *   64 or 128 the contraction
 *   runs on the tcgen05 tensor cores (h_in rounded to bf16 as an operand,
 *   as the forward does with its entering states); otherwise in exact fp32
 *   on the CUDA cores.  Tokens whose decay from the shard start underflows
 *   to zero (A <= 0) are left untouched.  workspace: >= the size
 *   ssd_state_correction_workspace_size reports (NULL only when that is 0).
 */
SSD_API ssd_status_t ssd_seq_logdecay(const float* dt, const float* A, float* logdecay,
                                      const ssd_dims_t* dims, void* stream);
SSD_API ssd_status_t ssd_state_exchange_combine(const float* local_final, const float* logdecay,
                                                const float* init, int rank, int nranks,
                                                float* h_in, const ssd_dims_t* dims,
                                                void* stream);
SSD_API ssd_status_t ssd_state_correction_workspace_size(const ssd_dims_t* dims,
                                                         ssd_dtype_t dtype, size_t* bytes);
SSD_API ssd_status_t ssd_state_correction_fwd(const float* h_in, const float* dt, const float* A,
                                              const void* C, void* y, float* final_states,
                                              const ssd_dims_t* dims, ssd_dtype_t dtype,
                                              void* workspace, size_t workspace_bytes,
                                              void* stream);

/*
 * Reports, and clears, a device-side wait that gave up in an earlier call on
 * the current device: the tensor-core kernels bound every wait, and one that
 * runs out records SSD_ERR_TIMEOUT in a device status word and ends the
 * kernel cleanly (its outputs are then incomplete).  Synchronises `stream`.
 * Returns SSD_OK if no wait gave up, SSD_ERR_TIMEOUT if one did.
 */
SSD_API ssd_status_t ssd_poll_device_status(void* stream);

/*
 * ssd_state_walk_fwd -- steps (2) and (3) fused: one CTA per (batch, head
 * pair) walks the chunks in order keeping the running fp32 state and each
 * chunk's contribution on chip (tensor memory), and writes only prev_states
 * (b,T,H,P,N) bf16 -- the state entering each chunk, same contents as
 * ssd_state_passing_fwd's -- and, if final_states is non-NULL, the fp32
 * state after the last chunk.  ssd_chunk_scan_fwd runs it (followed by
 * ssd_chunk_output_fwd's kernel) whenever ssd_chunk_scan_fwd_data_flow
 * reports SSD_FLOW_WALK_OUTPUT.  Covers the tensor-core sizes only
 * (SSD_BF16, chunk_size 128 or 256, headdim 64, 128, 192 or 256, dstate 64
 * or 128, any number of heads per group); other sizes return
 * SSD_ERR_UNSUPPORTED.
 */
SSD_API ssd_status_t ssd_state_walk_fwd(const void* x, const float* dt, const float* A,
                                        const void* B, const float* init_states,
                                        void* prev_states, float* final_states, int chunk_size,
                                        const ssd_dims_t* dims, ssd_dtype_t dtype, void* stream);

/*
 * Test hook for the failure path of the bounded device-side waits: launches
 * one CTA that waits on an mbarrier nothing ever arrives at, giving up after
 * at most `polls` polls (1 .. 2^20), so it records SSD_ERR_TIMEOUT in the
 * device status word exactly as a kernel whose wait ran out would.  The wait
 * always ends; nothing faults or hangs.  Read the result with
 * ssd_poll_device_status.
 */
SSD_API ssd_status_t ssd_debug_expire_wait(unsigned int polls, void* stream);

/* Which kernel family ssd_chunk_scan_fwd uses for these sizes:
 * 1 = tcgen05 tensor-core kernels, 0 = SIMT fp32 kernels, -1 = rejected.
 * The tensor cores take SSD_BF16 with headdim 32, 64, 128, 192 or 256 (a
 * head of headdim 64 k runs as k heads of 64 sharing dt, A, D; one of 32 as
 * a head of 64 whose other 32 columns are zero, its internal states padded
 * to 64 rows), dstate 64 or 128, any number of heads per group and any
 * chunk_size; everything else (and all of SSD_F32, whose 1e-4 bound rules
 * out bf16 operands) runs exact fp32.  The step entry points
 * (ssd_chunk_state_fwd, ssd_chunk_output_fwd, ssd_state_walk_fwd), whose
 * state buffers are the caller's, take the tensor cores for headdim 64 k
 * only. */
SSD_API int ssd_chunk_scan_fwd_uses_tensor_cores(const ssd_dims_t* dims, int chunk_size,
                                         ssd_dtype_t dtype);

/* Which data flow ssd_chunk_scan_fwd takes for these sizes (decided from the
 * sizes alone; the workspace size follows from it):
 *   SSD_FLOW_WALK_OUTPUT_FUSED  the same two parts in one launch: walkers
 *                            of two or four heads and output tiles side by
 *                            side, an output tile starting once the walkers
 *                            have written the states entering its chunk (8
 *                            chunks or more and at most 160 walkers; a memset
 *                            of the workspace's scheduling counters comes
 *                            first);
 *   SSD_FLOW_WALK_OUTPUT     state walk (steps 2+3 on chip, entering states
 *                            written in bf16) then the tensor-core output
 *                            kernel (steps 1+4): two launches;
 *   SSD_FLOW_TC_THREE_KERNEL tensor-core chunk states (fp32, in the
 *                            workspace), the state pass, the tensor-core
 *                            output kernel: three launches;
 *   SSD_FLOW_SIMT            the same three steps as exact-fp32 SIMT kernels;
 *   -1                       the sizes are rejected.
 * The walk is taken when there are enough (batch, head pair) walkers to
 * cover the GPU and enough chunks per walker (few long sequences keep the
 * three-kernel flow, whose state pass parallelises over state elements). */
#define SSD_FLOW_SIMT 0
#define SSD_FLOW_TC_THREE_KERNEL 1
#define SSD_FLOW_WALK_OUTPUT 2
#define SSD_FLOW_WALK_OUTPUT_FUSED 3
SSD_API int ssd_chunk_scan_fwd_data_flow(const ssd_dims_t* dims, int chunk_size,
                                         ssd_dtype_t dtype);

/*
 * ssd_chunk_scan_fwd with the data flow chosen by the caller: `flow` is one
 * of the SSD_FLOW_* values above, or -1 for the library's own choice (what
 * ssd_chunk_scan_fwd does).  Every flow computes the same result up to
 * rounding; SSD_FLOW_SIMT covers every size, the tensor-core flows the
 * sizes ssd_chunk_scan_fwd_uses_tensor_cores accepts.  A flow that does not
 * cover the sizes returns
 * SSD_ERR_UNSUPPORTED, an unknown one SSD_ERR_INVALID_ARG.  The workspace
 * must hold ssd_chunk_scan_fwd_flow_workspace_size(.., flow, ..) bytes.
 * For benchmarks and tests that compare the flows.
 */
SSD_API ssd_status_t ssd_chunk_scan_fwd_flow_workspace_size(const ssd_dims_t* dims,
                                                            int chunk_size, ssd_dtype_t dtype,
                                                            int flow, size_t* bytes);
SSD_API ssd_status_t ssd_chunk_scan_fwd_with_flow(const void* x, const float* dt, const float* A,
                                                  const void* B, const void* C, const float* D,
                                                  int chunk_size, const float* init_states,
                                                  void* y, float* final_states,
                                                  const ssd_dims_t* dims, ssd_dtype_t dtype,
                                                  void* workspace, size_t workspace_bytes,
                                                  void* stream, int flow);

#ifdef __cplusplus
}
#endif
#endif /* SSD_B200_H */
