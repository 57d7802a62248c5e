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

// ---------------------------------------------------------------- several steps, one launch
// `steps` successive tokens of one layer in one launch (the device-side counterpart of a
// generation loop that advances the cache with no host round trip per token, when the
// tokens' inputs are on the device already).  One CTA per (b, h) keeps that unit's state in
// registers for all the steps -- warp w holds rows w RPW .. w RPW + RPW - 1, lane j the
// 16-byte quad j of a row -- so the state is read once and written once, and the next
// step's inputs are loaded while this step is computed.  Each row's arithmetic is the
// single step's, operation for operation, so the results equal `steps` launches of
// decode_step_kernel bit for bit.  Inputs and outputs are [steps][...] arrays of the
// single step's layouts.
template <typename T, int RPW>
__global__ void __launch_bounds__(kDecodeThreads, RPW <= 8 ? 2 : 1)
decode_steps_kernel(float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
                    const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
                    const float* __restrict__ D, T* __restrict__ y, int steps, int batch, int nheads,
                    int headdim, int ngroups, int dstate)
{
    const int unit = blockIdx.x;
    const int b = unit / nheads;
    const int h = unit - b * nheads;
    const int g = h / (nheads / ngroups);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const bool qon = lane < (dstate >> 2);             // this lane's quad exists (dstate <= 128)
    const int p0 = warp * RPW;
    const size_t units = (size_t)batch * nheads;
    const float Ah = A[h], Dh = D[h];

    float4 s[RPW];
    float* S = state + (size_t)unit * headdim * dstate;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
        if (p0 + r < headdim && qon) s[r] = *reinterpret_cast<const float4*>(S + (size_t)(p0 + r) * dstate + 4 * lane);

    // the inputs of step k: dt, B_t and C_t (this lane's quad), x of this warp's rows
    auto load_step = [&](int k, float& dtv, float4& bq, float4& cq, float (&xv)[RPW]) {
        dtv = dt[(size_t)k * units + unit];
        const size_t bc = ((size_t)k * batch * ngroups + (size_t)b * ngroups + g) * dstate;
        bq = qon ? load4<T>(Bm + bc + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        cq = qon ? load4<T>(Cm + bc + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        const T* xr = x + ((size_t)k * units + unit) * headdim;
#pragma unroll
        for (int r = 0; r < RPW; ++r) xv[r] = p0 + r < headdim ? Elem<T>::load(xr + p0 + r) : 0.f;
    };
    float dtn = 0.f, xn[RPW];
    float4 bn, cn;
    if (steps > 0) load_step(0, dtn, bn, cn, xn);
    for (int k = 0; k < steps; ++k) {
        const float dtv = dtn;
        const float4 bq = bn, cq = cn;
        float xv[RPW];
#pragma unroll
        for (int r = 0; r < RPW; ++r) xv[r] = xn[r];
        if (k + 1 < steps) load_step(k + 1, dtn, bn, cn, xn);
        const float a = expf(dtv * Ah);                // fp32 decay exponent
        T* yr = y + ((size_t)k * units + unit) * headdim;
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int p = p0 + r;
            if (p >= headdim) break;                   // warp-uniform
            const float dx = dtv * xv[r];
            float acc = 0.f;
            if (qon) {
                float4 v = s[r];
                v.x = fmaf(a, v.x, dx * bq.x);
                v.y = fmaf(a, v.y, dx * bq.y);
                v.z = fmaf(a, v.z, dx * bq.z);
                v.w = fmaf(a, v.w, dx * bq.w);
                acc = fmaf(cq.x, v.x, acc);
                acc = fmaf(cq.y, v.y, acc);
                acc = fmaf(cq.z, v.z, acc);
                acc = fmaf(cq.w, v.w, acc);
                s[r] = v;
            }
            acc = warp_sum(acc);
            if (lane == 0) Elem<T>::store(yr + p, fmaf(Dh, xv[r], acc));
        }
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r)
        if (p0 + r < headdim && qon) *reinterpret_cast<float4*>(S + (size_t)(p0 + r) * dstate + 4 * lane) = s[r];
}

// Shapes whose state does not fit in registers: the single step's body once per step, still
// one launch (each CTA owns its unit's state, so the steps need no synchronisation).
template <typename T, int QPL, int ROWS>
__global__ void __launch_bounds__(kDecodeThreads, QPL == 1 ? 4 : 2)
decode_steps_loop_kernel(float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
                         const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
                         const float* __restrict__ D, T* __restrict__ y, int steps, int batch, int nheads,
                         int headdim, int ngroups, int dstate)
{
    const size_t units = (size_t)batch * nheads;
    for (int k = 0; k < steps; ++k)
        decode_unit<T, QPL, ROWS>(state, x + (size_t)k * units * headdim, dt + (size_t)k * units, A,
                                  Bm + (size_t)k * batch * ngroups * dstate, Cm + (size_t)k * batch * ngroups * dstate,
                                  D, y + (size_t)k * units * headdim, blockIdx.x, nheads, headdim, ngroups, dstate);
}

template <typename T>
cudaError_t launch_steps_dtype(const Dims& d, int steps, float* state, const void* x, const float* dt,
                               const float* A, const void* B, const void* C, const float* D, void* y,
                               cudaStream_t s)
{
    const unsigned grid = (unsigned)(d.batch * d.nheads);
    const T* xt = static_cast<const T*>(x);
    const T* Bt = static_cast<const T*>(B);
    const T* Ct = static_cast<const T*>(C);
    T* yt = static_cast<T*>(y);
    if (d.dstate <= 128 && d.headdim <= 64)
        decode_steps_kernel<T, 8><<<grid, kDecodeThreads, 0, s>>>(state, xt, dt, A, Bt, Ct, D, yt, steps, d.batch,
                                                                  d.nheads, d.headdim, d.ngroups, d.dstate);
    else if (d.dstate <= 128)
        decode_steps_kernel<T, 16><<<grid, kDecodeThreads, 0, s>>>(state, xt, dt, A, Bt, Ct, D, yt, steps, d.batch,
                                                                   d.nheads, d.headdim, d.ngroups, d.dstate);
    else if (d.dstate <= 256)
        decode_steps_loop_kernel<T, 2, 4><<<grid, kDecodeThreads, 0, s>>>(state, xt, dt, A, Bt, Ct, D, yt, steps,
                                                                          d.batch, d.nheads, d.headdim, d.ngroups,
                                                                          d.dstate);
    else
        decode_steps_loop_kernel<T, 4, 2><<<grid, kDecodeThreads, 0, s>>>(state, xt, dt, A, Bt, Ct, D, yt, steps,
                                                                          d.batch, d.nheads, d.headdim, d.ngroups,
                                                                          d.dstate);
    return cudaGetLastError();
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

cudaError_t launch_decode_steps(const Dims& d, ssd_dtype_t dtype, int steps, float* state, const void* x,
                                const float* dt, const float* A, const void* B, const void* C, const float* D,
                                void* y, cudaStream_t s)
{
    if (d.batch == 0 || steps == 0) return cudaSuccess;
    if (dtype == SSD_F32) return launch_steps_dtype<float>(d, steps, state, x, dt, A, B, C, D, y, s);
    return launch_steps_dtype<__nv_bfloat16>(d, steps, state, x, dt, A, B, C, D, y, s);
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
