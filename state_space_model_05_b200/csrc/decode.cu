// One-token SSD decode step over the O(1) state cache, in place.
//
// "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching
// for Inference", section "2. Metodologia": the cache holds one fixed-size state
// per (batch, head) and each generated token advances it on the device with no
// host round trip.  Per (b, h):
//     a = exp(dt_t * A_h);  H <- a H + dt_t x_t B_t^T;  y_t = H C_t + D_h x_t
// with H stored [headdim][dstate] (dstate innermost).
//
// The step is bound by HBM: every state element is read once and written once
// (8 bytes) for about five flops.  Design: one CTA of 8 warps per (b, h); each
// warp owns consecutive state rows (one row = dstate fp32 = 512 B at N=128) and
// issues ROWS 16-byte row loads before using any of them.  At dstate <= 128 four
// CTAs stay resident per SM (<= 64 registers, ROWS = 4): measured on B200 this
// keeps more bytes in flight than fewer, larger batches per thread.  B_t and C_t
// are read once per CTA into registers (lane j holds elements 4j..4j+3).  The y reduction along dstate is a
// warp shuffle tree; the state is written back with 16-byte stores.
#include "common.cuh"

namespace ssd {

namespace {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeWarps = kDecodeThreads / 32;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One (b, h) unit of the step, by one CTA.
// QPL: float4 quads of a state row per lane (dstate <= 128 * QPL).
// ROWS: rows a warp holds in flight at once.
template <typename T, int QPL, int ROWS>
__device__ __forceinline__ void decode_unit(float* __restrict__ state, const T* __restrict__ x,
                                            const float* __restrict__ dt, const float* __restrict__ A,
                                            const T* __restrict__ Bm, const T* __restrict__ Cm,
                                            const float* __restrict__ D, T* __restrict__ y, int unit,
                                            int nheads, int headdim, int ngroups, int dstate,
                                            const float* __restrict__ dt_bias = nullptr, int dt_softplus = 0)
{
    const int b = unit / nheads;
    const int h = unit - b * nheads;
    const int g = h / (nheads / ngroups);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nq = dstate >> 2;                        // quads per row

    const float dtv = dt_value(dt[unit], dt_bias, dt_softplus, h);
    const float a = expf(dtv * A[h]);                  // fp32 decay exponent
    const float Dh = D[h];

    const T* Bv = Bm + (size_t)(b * ngroups + g) * dstate;
    const T* Cv = Cm + (size_t)(b * ngroups + g) * dstate;
    float4 bq[QPL], cq[QPL];
#pragma unroll
    for (int q = 0; q < QPL; ++q) {
        const int j = lane + 32 * q;
        if (j < nq) {
            bq[q] = load4<T>(Bv + 4 * j);
            cq[q] = load4<T>(Cv + 4 * j);
        } else {
            bq[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            cq[q] = bq[q];
        }
    }

    float* S = state + (size_t)unit * headdim * dstate;
    const T* xr = x + (size_t)unit * headdim;
    T* yr = y + (size_t)unit * headdim;

    for (int p0 = warp * ROWS; p0 < headdim; p0 += kDecodeWarps * ROWS) {
        float4 s[ROWS][QPL];
        float xv[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            const int p = p0 + r;
            xv[r] = 0.f;
            if (p < headdim) {
                xv[r] = Elem<T>::load(xr + p);
#pragma unroll
                for (int q = 0; q < QPL; ++q) {
                    const int j = lane + 32 * q;
                    if (j < nq) s[r][q] = *reinterpret_cast<const float4*>(S + (size_t)p * dstate + 4 * j);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            const int p = p0 + r;
            if (p >= headdim) break;                   // warp-uniform
            const float dx = dtv * xv[r];
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < QPL; ++q) {
                const int j = lane + 32 * q;
                if (j < nq) {
                    float4 v = s[r][q];
                    v.x = fmaf(a, v.x, dx * bq[q].x);
                    v.y = fmaf(a, v.y, dx * bq[q].y);
                    v.z = fmaf(a, v.z, dx * bq[q].z);
                    v.w = fmaf(a, v.w, dx * bq[q].w);
                    acc = fmaf(cq[q].x, v.x, acc);
                    acc = fmaf(cq[q].y, v.y, acc);
                    acc = fmaf(cq[q].z, v.z, acc);
                    acc = fmaf(cq[q].w, v.w, acc);
                    *reinterpret_cast<float4*>(S + (size_t)p * dstate + 4 * j) = v;
                }
            }
            acc = warp_sum(acc);
            if (lane == 0) Elem<T>::store(yr + p, fmaf(Dh, xv[r], acc));
        }
    }
}

template <typename T, int QPL, int ROWS>
__global__ void __launch_bounds__(kDecodeThreads, QPL == 1 ? 4 : 2)
decode_step_kernel(float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
                   const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
                   const float* __restrict__ D, T* __restrict__ y, int nheads, int headdim,
                   int ngroups, int dstate, const float* __restrict__ dt_bias, int dt_softplus)
{
    decode_unit<T, QPL, ROWS>(state, x, dt, A, Bm, Cm, D, y, blockIdx.x, nheads, headdim, ngroups, dstate,
                              dt_bias, dt_softplus);
}

// Every layer of a stack in one launch: blockIdx.y is the layer, whose tensors come from
// the table.  A layer entry with a null or misaligned pointer is skipped and recorded.
template <typename T, int QPL, int ROWS>
__global__ void __launch_bounds__(kDecodeThreads, QPL == 1 ? 4 : 2)
decode_layers_kernel(const ssd_decode_layer_t* __restrict__ layers, int nheads, int headdim,
                     int ngroups, int dstate, int* err)
{
    const ssd_decode_layer_t L = layers[blockIdx.y];
    const uintptr_t any = reinterpret_cast<uintptr_t>(L.state) | reinterpret_cast<uintptr_t>(L.x_t) |
                          reinterpret_cast<uintptr_t>(L.dt_t) | reinterpret_cast<uintptr_t>(L.A) |
                          reinterpret_cast<uintptr_t>(L.B_t) | reinterpret_cast<uintptr_t>(L.C_t) |
                          reinterpret_cast<uintptr_t>(L.D) | reinterpret_cast<uintptr_t>(L.y_t);
    if (!L.state || !L.x_t || !L.dt_t || !L.A || !L.B_t || !L.C_t || !L.D || !L.y_t) {
        if (threadIdx.x == 0) record_error(err, SSD_ERR_NULL);
        return;
    }
    if (any & 15u) {
        if (threadIdx.x == 0) record_error(err, SSD_ERR_ALIGN);
        return;
    }
    decode_unit<T, QPL, ROWS>(L.state, static_cast<const T*>(L.x_t), L.dt_t, L.A,
                              static_cast<const T*>(L.B_t), static_cast<const T*>(L.C_t), L.D,
                              static_cast<T*>(L.y_t), blockIdx.x, nheads, headdim, ngroups, dstate);
}

template <typename T, int QPL, int ROWS>
cudaError_t launch_decode_t(const Dims& d, float* state, const void* x, const float* dt,
                            const float* A, const void* B, const void* C, const float* D, void* y,
                            cudaStream_t s)
{
    const unsigned grid = (unsigned)(d.batch * d.nheads);
    decode_step_kernel<T, QPL, ROWS><<<grid, kDecodeThreads, 0, s>>>(
        state, static_cast<const T*>(x), dt, A, static_cast<const T*>(B), static_cast<const T*>(C),
        D, static_cast<T*>(y), d.nheads, d.headdim, d.ngroups, d.dstate, d.dt_bias, d.dt_softplus);
    return cudaGetLastError();
}

template <typename T, int QPL, int ROWS>
cudaError_t launch_layers_t(const Dims& d, const ssd_decode_layer_t* layers, int n_layers, cudaStream_t s)
{
    const dim3 grid((unsigned)(d.batch * d.nheads), (unsigned)n_layers);
    decode_layers_kernel<T, QPL, ROWS><<<grid, kDecodeThreads, 0, s>>>(layers, d.nheads, d.headdim, d.ngroups,
                                                                      d.dstate, device_error_word());
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_layers_dtype(const Dims& d, const ssd_decode_layer_t* layers, int n_layers, cudaStream_t s)
{
    if (d.dstate <= 128) return launch_layers_t<T, 1, 4>(d, layers, n_layers, s);
    if (d.dstate <= 256) return launch_layers_t<T, 2, 4>(d, layers, n_layers, s);
    if (d.dstate <= 512) return launch_layers_t<T, 4, 2>(d, layers, n_layers, s);
    return cudaErrorInvalidValue;   // rejected earlier by argument validation
}

template <typename T>
cudaError_t launch_decode_dtype(const Dims& d, float* state, const void* x, const float* dt,
                                const float* A, const void* B, const void* C, const float* D,
                                void* y, cudaStream_t s)
{
    if (d.dstate <= 128) return launch_decode_t<T, 1, 4>(d, state, x, dt, A, B, C, D, y, s);
    if (d.dstate <= 256) return launch_decode_t<T, 2, 4>(d, state, x, dt, A, B, C, D, y, s);
    if (d.dstate <= 512) return launch_decode_t<T, 4, 2>(d, state, x, dt, A, B, C, D, y, s);
    return cudaErrorInvalidValue;   // rejected earlier by argument validation
}

}  // namespace

cudaError_t launch_decode_layers(const Dims& d, ssd_dtype_t dtype, const ssd_decode_layer_t* layers,
                                 int n_layers, cudaStream_t s)
{
    if (d.batch == 0 || n_layers == 0) return cudaSuccess;
    if (dtype == SSD_F32) return launch_layers_dtype<float>(d, layers, n_layers, s);
    return launch_layers_dtype<__nv_bfloat16>(d, layers, n_layers, s);
}

cudaError_t launch_decode(const Dims& d, ssd_dtype_t dtype, float* state, const void* x,
                          const float* dt, const float* A, const void* B, const void* C,
                          const float* D, void* y, cudaStream_t s)
{
    if (d.batch == 0) return cudaSuccess;
    if (dtype == SSD_F32) return launch_decode_dtype<float>(d, state, x, dt, A, B, C, D, y, s);
    return launch_decode_dtype<__nv_bfloat16>(d, state, x, dt, A, B, C, D, y, s);
}

}  // namespace ssd
