/*
 * ssd.h -- C ABI of the B200 (sm_100a) Mamba-2 state-space-duality (SSD) library.
 *
 * The operation.  "Compiler-First State Space Duality and Portable O(1)
 * Autoregressive Caching for Inference" (gist.science summary of arXiv
 * 2603.09555), section "2. Metodologia", describes the SSD layer of Mamba-2 as
 * a recurrence with per-head diagonal (scalar) decay that can be evaluated in
 * fixed-size chunks (prefill over the whole context) or one token at a time
 * against an O(1) state cache kept on the device (decode), with the decay
 * exponent taken in fp32.  For batch b, head h, group g = h / (nheads/ngroups):
 *
 *     a_t = exp(dt_t * A_h)
 *     H_t = a_t * H_{t-1} + dt_t * B_t x_t^T          (H: dstate x headdim)
 *     y_t = C_t^T H_t + D_h * x_t
 *
 * ssd_prefill evaluates it over `seqlen` tokens in chunks of `chunk_len`:
 * per chunk the inclusive cumulative sum of dt*A (the decay exponents), the
 * intra-chunk product (C B^T o L)(dt x) with the lower-triangular decay mask
 * L[t][s] = exp(sum_{r=s+1..t} dt_r A_h), the chunk's end state, the state
 * carried across chunks, and the carried state's contribution to y plus the
 * D skip.  ssd_decode_step advances the state cache by one token in place.
 * The result does not depend on chunk_len (up to rounding).
 *
 * Layouts (row-major, innermost last; all tensors contiguous):
 *     x, y         [batch][seqlen][nheads][headdim]       dtype `dtype`
 *     dt           [batch][seqlen][nheads]                fp32, dt > 0 (already softplus'd)
 *     A, D         [nheads]                               fp32
 *     B, C         [batch][seqlen][ngroups][dstate]       dtype `dtype`
 *     state        [batch][nheads][headdim][dstate]       fp32 (dstate innermost)
 *     decode x_t, y_t [batch][nheads][headdim]; dt_t [batch][nheads];
 *     decode B_t, C_t [batch][ngroups][dstate]
 *
 * Ownership: the caller allocates every buffer, device memory throughout
 * (including the prefill workspace); the library allocates no device memory
 * and keeps no state between calls besides one device error word per device
 * (and, only while kernel profiling is enabled, host-side event records).
 *
 * Streams and errors: every call is asynchronous on `stream` (a cudaStream_t
 * passed as void*, NULL = legacy default stream) and never synchronises.
 * Argument errors are detected on the host and returned before anything is
 * launched; nothing is written in that case.  A failed launch returns
 * SSD_ERR_CUDA.  A kernel that gives up a bounded wait records SSD_ERR_TIMEOUT
 * in the device error word, which ssd_device_status reads and clears.
 *
 * Requirements: nheads % ngroups == 0; headdim and dstate multiples of 8 with
 * headdim <= 128 and dstate <= 256 (prefill) or <= 512 (decode); chunk_len in
 * [1, 256]; every pointer 16-byte aligned; batch in [0, 65535] and seqlen >= 0
 * (batch 0 does nothing; seqlen 0 only copies init_state, or zeros, to
 * final_state).  Sizes outside these ranges return SSD_ERR_UNSUPPORTED or
 * SSD_ERR_SHAPE.  bf16 prefills with headdim 64, dstate 128 and chunk_len
 * 128 or 256 run on the tensor cores (tcgen05); every other shape runs the
 * same chunked algorithm on the CUDA cores in fp32.
 */
#ifndef SSD_H
#define SSD_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_NULL = 1,        /* a required pointer is NULL */
    SSD_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
    SSD_ERR_DTYPE = 3,       /* unknown dtype */
    SSD_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned */
    SSD_ERR_UNSUPPORTED = 5, /* valid, but not a shape this library implements */
    SSD_ERR_CUDA = 6,        /* a CUDA call or launch failed */
    SSD_ERR_TIMEOUT = 7,     /* a device-side bounded wait expired */
    SSD_ERR_WORKSPACE = 8    /* workspace missing or smaller than required */
} ssd_status_t;

/* Storage type of x, B, C and y (and of x_t, B_t, C_t, y_t for decode).
 * dt, A, D and the state are always fp32; accumulation is always fp32. */
typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype_t;

/* Version of this ABI (major * 100 + minor). */
int ssd_abi_version(void);

/* Human-readable name of a status code; never NULL. */
const char* ssd_status_string(ssd_status_t status);

/*
 * Bytes of device workspace ssd_prefill needs for these sizes (0 when the
 * sizes are invalid).  The workspace holds the per-chunk decay exponents and
 * the per-chunk states; its contents need no initialisation and are not
 * meaningful after the call.
 */
size_t ssd_prefill_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int ngroups,
                                   int dstate, int chunk_len, ssd_dtype_t dtype);

/*
 * Chunked prefill.  Reads x, dt, A, B, C, D (and init_state when non-NULL,
 * the state before the first token; NULL means zeros); writes y and
 * final_state (the state after the last token).  x, B, C and y are `dtype`;
 * y is rounded once to `dtype` from fp32.  `workspace` must hold at least
 * ssd_prefill_workspace_bytes(...) bytes of device memory.
 * init_state may be the same buffer as final_state (each state element is
 * read before it is written); otherwise no output may overlap any input.
 */
ssd_status_t ssd_prefill(const void* x, const float* dt, const float* A, const void* B,
                         const void* C, const float* D, const float* init_state, int batch,
                         int seqlen, int nheads, int headdim, int ngroups, int dstate,
                         int chunk_len, ssd_dtype_t dtype, void* y, float* final_state,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Which tensor-core kernels a batched bf16 prefill (headdim 64, dstate 128, chunk_len 128
 * or 256) runs, process-wide:
 *   SSD_PREFILL_TWO_PASS: a chunk-state walk writes each block's start state to the
 *     workspace, then a block-output kernel reads it back (one CTA per block and group
 *     of heads);
 *   SSD_PREFILL_FUSED: after a kernel forming G = C B^T per block, one kernel walks the
 *     128-token blocks of head pairs in order with the pairs' states in tensor memory and
 *     writes y and the final state (x read once; a state goes through global memory only
 *     where a pair's blocks are split between two CTAs).  It needs an even number of heads
 *     per group; other shapes take the two-pass kernels;
 *   SSD_PREFILL_AUTO (the default): the two-pass kernels, the faster of the two on every
 *     workload measured so far.
 * Both compute the same chunked algorithm with bf16 operands and fp32 accumulation; the
 * results agree to rounding.  Packed variable-length prefills always take the two-pass
 * kernels, other shapes the CUDA-core path.  The workspace size covers either.  Returns
 * SSD_ERR_SHAPE for an unknown value.  Not synchronised with calls in flight on other
 * host threads.
 */
typedef enum { SSD_PREFILL_AUTO = 0, SSD_PREFILL_FUSED = 1, SSD_PREFILL_TWO_PASS = 2 } ssd_prefill_path_t;
ssd_status_t ssd_set_prefill_path(ssd_prefill_path_t path);
ssd_prefill_path_t ssd_get_prefill_path(void);

/*
 * One decode step on the state cache, in place: each fp32 state row is read
 * once, decayed by exp(dt_t * A_h), given the rank-1 update dt_t B_t x_t^T,
 * reduced against C_t for y_t, and written back.  x_t, B_t, C_t, y_t are
 * `dtype`.  No host synchronisation; any number of steps may be queued or
 * captured in a CUDA graph.
 */
ssd_status_t ssd_decode_step(float* state, const void* x_t, const float* dt_t, const float* A,
                             const void* B_t, const void* C_t, const float* D, int batch,
                             int nheads, int headdim, int ngroups, int dstate, ssd_dtype_t dtype,
                             void* y_t, void* stream);

/*
 * `steps` successive decode steps of one layer in one launch, for tokens whose inputs are
 * already on the device: the O(1) cache advanced on the device by a loop with no host round
 * trip per token ("Compiler-First State Space Duality and Portable O(1) Autoregressive
 * Caching for Inference", section "2. Metodologia": the compiled generation loop).
 *   x, y: [steps][batch][nheads][headdim] (`dtype`); dt: [steps][batch][nheads] fp32;
 *   B, C: [steps][batch][ngroups][dstate] (`dtype`); A, D: [nheads] fp32; state in/out as
 *   for ssd_decode_step.  Step k uses the k-th slice of each input and writes the k-th slice
 *   of y.
 * The result equals `steps` calls of ssd_decode_step on the slices, bit for bit.  With
 * dstate <= 128 each (batch, head) state stays on chip for all the steps, so the state is
 * read once and written once per call instead of once per step.  steps = 0 does nothing;
 * steps < 0 is SSD_ERR_SHAPE; errors as for ssd_decode_step.
 */
ssd_status_t ssd_decode_steps(float* state, const void* x, const float* dt, const float* A,
                              const void* B, const void* C, const float* D, int steps, int batch,
                              int nheads, int headdim, int ngroups, int dstate, ssd_dtype_t dtype,
                              void* y, void* stream);

/*
 * ssd_prefill / ssd_decode_step with the dt pre-processing folded into the kernels: the dt
 * the recurrence uses is softplus(dt_raw + dt_bias[h]) (softplus(z) = log(1 + exp(z)); z
 * itself above 40), formed in double precision and rounded to fp32 once, so a caller
 * passes the projection's raw dt.
 * dt_raw has dt's layout; dt_bias is [nheads] fp32 (16-byte aligned) or NULL for no bias.
 * The pages feed the SSD a positive dt and say nothing of how it is produced; this is the
 * softplus parameterisation of dt the synthetic workloads use (dt = softplus(z + b_h)).
 * Everything else, including the workspace size, is as for the plain call.
 */
ssd_status_t ssd_prefill_dtraw(const void* x, const float* dt_raw, const float* dt_bias,
                               const float* A, const void* B, const void* C, const float* D,
                               const float* init_state, int batch, int seqlen, int nheads,
                               int headdim, int ngroups, int dstate, int chunk_len,
                               ssd_dtype_t dtype, void* y, float* final_state, void* workspace,
                               size_t workspace_bytes, void* stream);
ssd_status_t ssd_decode_step_dtraw(float* state, const void* x_t, const float* dt_raw_t,
                                   const float* dt_bias, const float* A, const void* B_t,
                                   const void* C_t, const float* D, int batch, int nheads,
                                   int headdim, int ngroups, int dstate, ssd_dtype_t dtype,
                                   void* y_t, void* stream);

/*
 * Packed variable-length prefill: nseq sequences laid end to end along one token axis, the
 * state reset at every sequence start.  Sequence i is tokens cu_seqlens[i] ..
 * cu_seqlens[i + 1] - 1 of x, dt, B, C and y, which have the layouts of ssd_prefill with
 * batch 1 and seqlen = total_tokens; it starts from init_states[i] (NULL: zeros) and ends in
 * final_states[i] ([nseq][nheads][headdim][dstate] fp32).  Equivalent to one ssd_prefill per
 * sequence, in one call; the pages' cache carries one state per sequence ("Compiler-First
 * State Space Duality ...", section "2. Metodologia"), and this is prefill of many cached
 * sequences at once.
 *   cu_seqlens: DEVICE array of nseq + 1 int32 offsets, read by the kernels: cu_seqlens[0]
 *   = 0, non-decreasing, cu_seqlens[nseq] = total_tokens (else SSD_ERR_SHAPE is recorded
 *   in the device error word and nothing is computed).  Empty sequences are allowed.
 * Sizes and dtypes as for ssd_prefill (the tensor-core path for bf16, headdim 64, dstate
 * 128, chunk_len 128 or 256; the CUDA-core path otherwise).  `workspace` must hold
 * ssd_prefill_varlen_workspace_bytes(...) bytes (0 when total_tokens is 0).
 */
size_t ssd_prefill_varlen_workspace_bytes(int nseq, int total_tokens, int nheads, int headdim,
                                          int ngroups, int dstate, int chunk_len, ssd_dtype_t dtype);
ssd_status_t ssd_prefill_varlen(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, const float* init_states,
                                const int* cu_seqlens, int nseq, int total_tokens, int nheads,
                                int headdim, int ngroups, int dstate, int chunk_len, ssd_dtype_t dtype,
                                void* y, float* final_states, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * One layer's tensors for ssd_decode_step_layers: the arguments of ssd_decode_step for
 * that layer (device pointers, layouts as there; every pointer 16-byte aligned).
 */
typedef struct {
    float* state;          /* [batch][nheads][headdim][dstate] fp32, in/out */
    const void* x_t;       /* [batch][nheads][headdim] dtype */
    const float* dt_t;     /* [batch][nheads] */
    const float* A;        /* [nheads] */
    const void* B_t;       /* [batch][ngroups][dstate] dtype */
    const void* C_t;       /* [batch][ngroups][dstate] dtype */
    const float* D;        /* [nheads] */
    void* y_t;             /* [batch][nheads][headdim] dtype */
} ssd_decode_layer_t;

/*
 * One decode step of every layer of a stack, in one launch: for each of the n_layers
 * entries of `layers` (a DEVICE array of ssd_decode_layer_t, read by the kernel), exactly
 * what ssd_decode_step does for that layer.  All layers share the sizes and dtype.  The
 * pages run the cache update inside one compiled on-device loop ("Compiler-First State
 * Space Duality ...", section "2. Metodologia"); this is that idea across layers: one
 * launch per token for the whole stack.  The sizes are checked on the host
 * (SSD_ERR_SHAPE/DTYPE, SSD_ERR_NULL for a NULL table); the entries are checked on the
 * device: an entry with a NULL or misaligned pointer is skipped and records
 * SSD_ERR_NULL / SSD_ERR_ALIGN in the device error word (ssd_device_status).  The layers'
 * state buffers must not overlap one another or any input.
 */
ssd_status_t ssd_decode_step_layers(const ssd_decode_layer_t* layers, int n_layers, int batch,
                                    int nheads, int headdim, int ngroups, int dstate,
                                    ssd_dtype_t dtype, void* stream);

/*
 * `steps` successive decode steps of every layer of a stack in one launch: the stack's O(1)
 * caches advanced by a device-side loop with no host round trip per token ("Compiler-First
 * State Space Duality and Portable O(1) Autoregressive Caching for Inference", section
 * "2. Metodologia"), for tokens whose per-layer inputs are already on the device.  Each of
 * the n_layers entries of `layers` (a DEVICE array, as for ssd_decode_step_layers) holds the
 * arguments of ssd_decode_steps for its layer: x_t, dt_t, B_t, C_t and y_t point at that
 * layer's [steps][...] arrays.  The result equals ssd_decode_steps on each layer (and so
 * `steps` calls of ssd_decode_step per layer) bit for bit.  Sizes are checked on the host
 * (SSD_ERR_SHAPE/DTYPE/UNSUPPORTED; steps < 0 or n_layers outside [0, 65535] is
 * SSD_ERR_SHAPE; SSD_ERR_NULL for a NULL table); entries on the device as for
 * ssd_decode_step_layers (a NULL or misaligned entry is skipped and recorded in the device
 * error word).  steps = 0 or n_layers = 0 does nothing.  No state buffer may overlap another
 * layer's buffers or any input.
 */
ssd_status_t ssd_decode_steps_layers(const ssd_decode_layer_t* layers, int n_layers, int steps, int batch,
                                     int nheads, int headdim, int ngroups, int dstate, ssd_dtype_t dtype,
                                     void* stream);

/*
 * Gated DeltaNet decode step (a second recurrent workload, on its own state cache):
 * "Persistent-State Dataflow Accelerator for Memory-Bound Linear Attention Decode on
 * FPGA", section 2.B.  Per (b, value head h), with query/key head hk = h / (heads_v /
 * heads_qk) (section 2.C: value heads grouped on shared query/key heads):
 *     dv = beta (v - gate S^T k);   S <- gate S + k dv^T;   out = S^T q  (updated S)
 * computed as one read pass and one write pass over S (out = gate S_old^T q + (q.k) dv).
 * The page leaves dv undefined; the gated delta rule above is the reading used.
 *   state  [batch][heads_v][dk][dv] fp32, in/out (dv innermost)
 *   q, k   [batch][heads_qk][dk] dtype;  v, out [batch][heads_v][dv] dtype
 *   gate, beta [batch][heads_v] fp32 (gate in (0, 1], beta in [0, 1] for a contracting
 *   update; any finite values are computed as given)
 * Requirements: heads_v % heads_qk == 0; dk a multiple of 8 up to 128; dv a multiple of
 * 4 up to 128 (else SSD_ERR_SHAPE / SSD_ERR_UNSUPPORTED); 16-byte aligned pointers.
 * Asynchronous on `stream`; the state buffer must not overlap any input or `out`.
 */
ssd_status_t ssd_gdn_decode_step(float* state, const void* q, const void* k, const void* v,
                                 const float* gate, const float* beta, int batch, int heads_qk,
                                 int heads_v, int dk, int dv, ssd_dtype_t dtype, void* out,
                                 void* stream);

/*
 * ssd_prefill without a workspace argument, for callers that may not allocate
 * device memory (a host framework's execution hook that must stay inside the
 * memory it planned, or code running during a CUDA stream capture, where
 * cudaMalloc would break the capture).  The paper has no counterpart to this
 * entry point; it is a deployment convenience.
 *
 * The workspace comes from a 64 MiB buffer built into the library's device
 * image (held by every GPU that loads the library until the process exits).
 * Sizes whose ssd_prefill_workspace_bytes exceeds 64 MiB return
 * SSD_ERR_WORKSPACE before anything is launched.  The first call on a device
 * looks up the buffer's device address (with that device current); make that
 * first call before any stream capture.  All calls share the one buffer:
 * calls that overlap on the GPU (e.g. on two streams) race and must be
 * serialised by the caller.  Nothing needs clearing between calls.
 * Everything else is as for ssd_prefill.
 */
ssd_status_t ssd_prefill_noalloc(const void* x, const float* dt, const float* A, const void* B,
                                 const void* C, const float* D, const float* init_state,
                                 int batch, int seqlen, int nheads, int headdim, int ngroups,
                                 int dstate, int chunk_len, ssd_dtype_t dtype, void* y,
                                 float* final_state, void* stream);

/*
 * Diagnostic: runs the library's bounded device waits against conditions that never
 * become true (an mbarrier nothing arrives on, a flag nothing sets), with short
 * limits.  Both waits expire, so after it the device error word holds SSD_ERR_TIMEOUT
 * (read it with ssd_device_status) and the CUDA context stays usable.  `scratch` is 3
 * ints of device memory: [0] is the flag, [1] and [2] receive 1 if the mbarrier wait,
 * respectively the flag wait, completed (0 when it gave up, as expected).
 */
ssd_status_t ssd_selftest_bounded_waits(int* scratch, void* stream);

/*
 * Synchronises `stream`, then reads and clears this device's error word.
 * Returns SSD_OK, SSD_ERR_TIMEOUT (a bounded wait expired in a kernel since
 * the last call), or SSD_ERR_CUDA when the stream reports a CUDA error.
 */
ssd_status_t ssd_device_status(void* stream);

/*
 * Kernel profiling (diagnostics; off by default).  While enabled, ssd_prefill
 * and ssd_decode_step record a CUDA event before and after each kernel they
 * launch, on the call's stream (so the events may also be captured in a CUDA
 * graph; they then re-record on every replay and a read reflects the latest
 * replay).  ssd_profile_read synchronises on
 * the recorded events and returns, per kernel name, the summed milliseconds
 * and the number of launches since the last ssd_profile_reset.  Not thread
 * safe; meant for benchmarks.
 */
void ssd_profile_enable(int on);
void ssd_profile_reset(void);
/* Writes up to max_kernels entries; returns the number written, or -1 on a
 * CUDA error.  `names` receives static strings owned by the library. */
int ssd_profile_read(int max_kernels, const char** names, double* total_ms, long long* launches);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H */
