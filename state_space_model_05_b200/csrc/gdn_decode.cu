// One-token Gated DeltaNet decode over the per-head state, in place.
//
// "Persistent-State Dataflow Accelerator for Memory-Bound Linear Attention Decode on
// FPGA", section 2.B: per value head the dk x dv state advances as
//     S_t = g S_{t-1} + k dv^T,   o_t = S_t^T q,   dv = beta (v - g S_{t-1}^T k)
// (the gated delta rule), and the identity S_t^T q = g S_{t-1}^T q + (q^T k) dv lets one
// read pass over S produce both S_{t-1}^T k and S_{t-1}^T q, after which one write pass
// stores S_t -- one read and one write of the state per token.  Section 2.C: value heads
// come in groups sharing one query/key head (head h reads query/key head h / (hv / hqk)).
//
// The step is bound by memory: 8 bytes of state traffic per element against ~6 flops.
// The columns of S are independent (each column's sums over the rows decide only that
// column), so one CTA of 4 warps takes one (b, value head, 64-column block); thread
// (row group rg, column quad c) owns rows 16 rg .. 16 rg + 15 of columns 4c .. 4c + 3,
// issues those 16 float4 loads before using any of them and keeps them in registers
// through the write pass.  The column sums of S^T k and S^T q cross the row groups
// through shared memory once.  Four such CTAs stay resident per SM.
#include "common.cuh"

namespace ssd {

namespace {

constexpr int kGdnThreads = 128;
constexpr int kGdnMaxDk = 128;
constexpr int kGdnMaxDv = 128;
constexpr int kGdnCols = 64;                               // state columns per CTA
constexpr int kColQuads = kGdnCols / 4;                    // 16
constexpr int kRowGroups = kGdnThreads / kColQuads;        // 8
constexpr int kGdnRows = kGdnMaxDk / kRowGroups;           // 16 rows per thread

template <typename T>
__global__ void __launch_bounds__(kGdnThreads, 4)
gdn_decode_kernel(float* __restrict__ state, const T* __restrict__ q, const T* __restrict__ k,
                  const T* __restrict__ v, const float* __restrict__ gate, const float* __restrict__ beta,
                  T* __restrict__ out, int hqk, int hv, int dk, int dv)
{
    __shared__ float sq[kGdnMaxDk], sk[kGdnMaxDk];
    __shared__ float4 red[2][kRowGroups][kColQuads];    // per-row-group partial S^T k and S^T q
    __shared__ float sqk;

    const int unit = blockIdx.x;                       // b * hv + h
    const int b = unit / hv, h = unit - b * hv;
    const int hk = h / (hv / hqk);
    const int tid = threadIdx.x, cq = tid % kColQuads, rg = tid / kColQuads;
    const int c0 = blockIdx.y * kGdnCols + 4 * cq;     // first of this thread's 4 columns
    const bool col = c0 < dv;

    const T* qh = q + ((size_t)b * hqk + hk) * dk;
    const T* kh = k + ((size_t)b * hqk + hk) * dk;
    for (int i = tid; i < dk; i += kGdnThreads) {
        sq[i] = Elem<T>::load(qh + i);
        sk[i] = Elem<T>::load(kh + i);
    }
    const float g = gate[unit], bt = beta[unit];

    // read pass: this thread's rows of its columns, all loads in flight before any use
    float* S = state + (size_t)unit * dk * dv;
    const int i0 = rg * kGdnRows;
    float4 s[kGdnRows];
#pragma unroll
    for (int r = 0; r < kGdnRows; ++r) {
        const int i = i0 + r;
        s[r] = (col && i < dk) ? *reinterpret_cast<const float4*>(S + (size_t)i * dv + c0)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();                                   // q, k in shared memory
    if (tid < 32) {
        float d = 0.f;
        for (int i = tid; i < dk; i += 32) d = fmaf(sq[i], sk[i], d);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (tid == 0) sqk = d;
    }
    float4 rk = make_float4(0.f, 0.f, 0.f, 0.f), rq = rk;
#pragma unroll
    for (int r = 0; r < kGdnRows; ++r) {
        const int i = i0 + r;
        const float ki = i < dk ? sk[i] : 0.f, qi = i < dk ? sq[i] : 0.f;
        rk.x = fmaf(s[r].x, ki, rk.x); rk.y = fmaf(s[r].y, ki, rk.y);
        rk.z = fmaf(s[r].z, ki, rk.z); rk.w = fmaf(s[r].w, ki, rk.w);
        rq.x = fmaf(s[r].x, qi, rq.x); rq.y = fmaf(s[r].y, qi, rq.y);
        rq.z = fmaf(s[r].z, qi, rq.z); rq.w = fmaf(s[r].w, qi, rq.w);
    }
    red[0][rg][cq] = rk;
    red[1][rg][cq] = rq;
    __syncthreads();
    if (!col) return;                                  // columns past dv

    // column sums over the row groups (every row group forms them for its own columns)
    float4 tk = make_float4(0.f, 0.f, 0.f, 0.f), tq = tk;
#pragma unroll
    for (int w = 0; w < kRowGroups; ++w) {
        const float4 a = red[0][w][cq], c = red[1][w][cq];
        tk.x += a.x; tk.y += a.y; tk.z += a.z; tk.w += a.w;
        tq.x += c.x; tq.y += c.y; tq.z += c.z; tq.w += c.w;
    }
    const float4 vv = load4<T>(v + (size_t)unit * dv + c0);
    float4 corr;                                       // dv = beta (v - g S^T k)
    corr.x = bt * (vv.x - g * tk.x);
    corr.y = bt * (vv.y - g * tk.y);
    corr.z = bt * (vv.z - g * tk.z);
    corr.w = bt * (vv.w - g * tk.w);

    // write pass: S_t = g S + k dv^T
#pragma unroll
    for (int r = 0; r < kGdnRows; ++r) {
        const int i = i0 + r;
        if (i < dk) {
            const float ki = sk[i];
            float4 n;
            n.x = fmaf(ki, corr.x, g * s[r].x);
            n.y = fmaf(ki, corr.y, g * s[r].y);
            n.z = fmaf(ki, corr.z, g * s[r].z);
            n.w = fmaf(ki, corr.w, g * s[r].w);
            *reinterpret_cast<float4*>(S + (size_t)i * dv + c0) = n;
        }
    }
    if (rg == 0) {                                     // o = g S^T q + (q^T k) dv
        const float qk = sqk;
        T* o = out + (size_t)unit * dv + c0;
        Elem<T>::store(o + 0, fmaf(qk, corr.x, g * tq.x));
        Elem<T>::store(o + 1, fmaf(qk, corr.y, g * tq.y));
        Elem<T>::store(o + 2, fmaf(qk, corr.z, g * tq.z));
        Elem<T>::store(o + 3, fmaf(qk, corr.w, g * tq.w));
    }
}

}  // namespace

bool gdn_sizes_supported(int dk, int dv)
{
    return dk >= 1 && dk <= kGdnMaxDk && dk % 8 == 0 && dv >= 4 && dv <= kGdnMaxDv && dv % 4 == 0;
}

cudaError_t launch_gdn_decode(ssd_dtype_t dtype, float* state, const void* q, const void* k,
                              const void* v, const float* gate, const float* beta, void* out,
                              int batch, int hqk, int hv, int dk, int dv, cudaStream_t s)
{
    if (batch == 0) return cudaSuccess;
    const dim3 grid((unsigned)(batch * hv), (unsigned)((dv + kGdnCols - 1) / kGdnCols));
    if (dtype == SSD_F32)
        gdn_decode_kernel<float><<<grid, kGdnThreads, 0, s>>>(
            state, static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
            gate, beta, static_cast<float*>(out), hqk, hv, dk, dv);
    else
        gdn_decode_kernel<__nv_bfloat16><<<grid, kGdnThreads, 0, s>>>(
            state, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), gate, beta, static_cast<__nv_bfloat16*>(out), hqk, hv,
            dk, dv);
    return cudaGetLastError();
}

}  // namespace ssd
