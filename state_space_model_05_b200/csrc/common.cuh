// Shared internals of the SSD library (device helpers, launch declarations).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

// Device error word (one per device, defined in api.cu): kernels that wait set it
// when a bounded wait expires; ssd_device_status reads and clears it.  Kernels get
// its address as an argument.
int* device_error_word();   // host: address on the current device (nullptr on failure)

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// ---- element loads/stores for the two storage types -------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// Four consecutive elements as fp32 (16-byte load for fp32, 8-byte for bf16).
template <typename T> __device__ __forceinline__ float4 load4(const T* p);
template <> __device__ __forceinline__ float4 load4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <> __device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    float4 r;
    r.x = __uint_as_float(u.x << 16);
    r.y = __uint_as_float(u.x & 0xFFFF0000u);
    r.z = __uint_as_float(u.y << 16);
    r.w = __uint_as_float(u.y & 0xFFFF0000u);
    return r;
}

// ---- problem description passed to every launcher ---------------------------------
struct Dims {
    int batch, seqlen, nheads, headdim, ngroups, dstate, chunk_len, nchunks;
    // dt as the kernels use it: dt_in itself, or with dt_softplus softplus(dt_in + dt_bias[h])
    // (dt_bias may be null: no bias)
    const float* dt_bias = nullptr;
    int dt_softplus = 0;
    // Packed variable-length mode (tensor-core path): batch 1, nseq sequences end to end
    // along seqlen; nchunks is then an upper bound on the blocks of all sequences.
    int nseq = 0;                   // 0: batched mode
    const int* cu_seqlens = nullptr;  // device [nseq + 1] token offsets
    const int* vl_first = nullptr;    // device [nseq + 1] first block of each sequence, then the total
    const int* vl_seq = nullptr;      // device [nchunks] sequence of each block, -1 past the total
};

// Rows of block kb in packed variable-length mode: false if kb holds no tokens.
__device__ __forceinline__ bool varlen_block(const int* cu, const int* first, const int* seqof, int kb,
                                             int Q, int* seq, int* t0, int* len) {
    const int s = seqof[kb];
    if (s < 0) return false;
    *seq = s;
    *t0 = cu[s] + (kb - first[s]) * Q;
    *len = min(Q, cu[s + 1] - *t0);
    return true;
}

// The dt a kernel uses for head h from the dt input value `in`.  With dt_softplus the sum
// in + dt_bias[h] and softplus(z) = log(1 + exp(z)) (z itself above 40) are formed in
// double precision and rounded to fp32 once: for small dt, softplus(z) ~ exp(z) turns an
// fp32 rounding of z into a relative error of dt that the decay exponents then accumulate.
__device__ __forceinline__ float dt_value(float in, const float* dt_bias, int dt_softplus, int h) {
    if (!dt_softplus) return in;
    const double z = (double)in + (dt_bias ? (double)dt_bias[h] : 0.0);
    return (float)(z > 40.0 ? z : log1p(exp(z)));
}

// Workspace layout of the CUDA-core chunked prefill (offsets from the workspace base).
struct PrefillWorkspace {
    float* lam;      // [batch][nheads][nchunks][2][chunk_len] inclusive cumsum of dt*A, summed
                     //   in double and kept as two floats (hi = fl(Lam), lo = fl(Lam - hi))
    float* states;   // [batch][nheads][nchunks][headdim][dstate]
};
size_t prefill_workspace_layout(const Dims& d, void* base, PrefillWorkspace* ws);

constexpr int kMaxChunk = 256;               // largest chunk length Q

// ---- launchers (return cudaGetLastError() of their launches) -----------------------
// Gated DeltaNet decode step (gdn_decode.cu).
bool gdn_sizes_supported(int dk, int dv);
cudaError_t launch_gdn_decode(ssd_dtype_t dtype, float* state, const void* q, const void* k,
                              const void* v, const float* gate, const float* beta, void* out,
                              int batch, int hqk, int hv, int dk, int dv, cudaStream_t s);

// Every layer of a stack, one launch (layers: device array of n_layers entries).
cudaError_t launch_decode_layers(const Dims& d, ssd_dtype_t dtype, const ssd_decode_layer_t* layers,
                                 int n_layers, cudaStream_t s);

// `steps` successive decode steps of every layer of a table, one launch.
cudaError_t launch_decode_steps_layers(const Dims& d, ssd_dtype_t dtype, const ssd_decode_layer_t* layers,
                                       int n_layers, int steps, cudaStream_t s);

// `steps` successive decode steps in one launch (inputs and outputs [steps][...]).
cudaError_t launch_decode_steps(const Dims& d, ssd_dtype_t dtype, int steps, float* state, const void* x,
                                const float* dt, const float* A, const void* B, const void* C, const float* D,
                                void* y, cudaStream_t s);

cudaError_t launch_decode(const Dims& d, ssd_dtype_t dtype, float* state, const void* x,
                          const float* dt, const float* A, const void* B, const void* C,
                          const float* D, void* y, cudaStream_t s);

// Lambda (within-chunk cumulative sum of dt A) for every (b, h, chunk) row of `fac`:
// [b][h][c][2][Q] (Lambda summed in double, as hi and lo floats), or with `extras`
// [b][h][c][4][Q] holding Lambda (fp32), dt and the two column
// factors per 32-token sub-block (exp(Lam_last - Lam_s) dt_s, exp(Lam_first - Lam_s) dt_s;
// Q a multiple of 32).  Optionally the chunk-state weights exp(Lam_end - Lam_s) dt_s followed
// by exp(Lam_end) and three zeros ([b][h][c][Q + 4]), and an fp16 copy of a bf16 B.  Null
// outputs are skipped.
cudaError_t launch_chunk_cumsum(const Dims& d, const float* dt, const float* A, float* fac,
                                bool extras, float* wts, const void* b_bf16, void* b_f16,
                                cudaStream_t s);
cudaError_t launch_chunk_state_simt(const Dims& d, ssd_dtype_t dtype, const void* x,
                                    const float* dt, const void* B, const float* lam,
                                    float* states, cudaStream_t s);
cudaError_t launch_state_scan(const Dims& d, const float* lam, float* states,
                              const float* init_state, float* final_state, cudaStream_t s);
cudaError_t launch_chunk_output_simt(const Dims& d, ssd_dtype_t dtype, const void* x,
                                     const float* dt, const void* B, const void* C,
                                     const float* D, const float* lam, const float* states,
                                     void* y, cudaStream_t s);
cudaError_t launch_copy_state(const Dims& d, const float* init_state, float* final_state,
                              cudaStream_t s);

}  // namespace ssd
