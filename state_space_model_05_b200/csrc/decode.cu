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
#include "prefill_tc.h"
#include "ptx.cuh"

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

// A layer table entry is used when none of its pointers is null and all are 16-byte
// aligned; otherwise the CTA skips it and thread 0 records SSD_ERR_NULL / SSD_ERR_ALIGN.
__device__ __forceinline__ bool layer_entry_ok(const ssd_decode_layer_t& L, int* err)
{
    const uintptr_t any = reinterpret_cast<uintptr_t>(L.state) | reinterpret_cast<uintptr_t>(L.x_t) |
                          reinterpret_cast<uintptr_t>(L.dt_t) | reinterpret_cast<uintptr_t>(L.A) |
                          reinterpret_cast<uintptr_t>(L.B_t) | reinterpret_cast<uintptr_t>(L.C_t) |
                          reinterpret_cast<uintptr_t>(L.D) | reinterpret_cast<uintptr_t>(L.y_t);
    if (!L.state || !L.x_t || !L.dt_t || !L.A || !L.B_t || !L.C_t || !L.D || !L.y_t) {
        if (threadIdx.x == 0) record_error(err, SSD_ERR_NULL);
        return false;
    }
    if (any & 15u) {
        if (threadIdx.x == 0) record_error(err, SSD_ERR_ALIGN);
        return false;
    }
    return true;
}

// Every layer of a stack in one launch: blockIdx.y is the layer, whose tensors come from
// the table.  A layer entry with a null or misaligned pointer is skipped and recorded.
template <typename T, int QPL, int ROWS>
__global__ void __launch_bounds__(kDecodeThreads, QPL == 1 ? 4 : 2)
decode_layers_kernel(const ssd_decode_layer_t* __restrict__ layers, int nheads, int headdim,
                     int ngroups, int dstate, int* err)
{
    const ssd_decode_layer_t L = layers[blockIdx.y];
    if (!layer_entry_ok(L, err)) return;
    decode_unit<T, QPL, ROWS>(L.state, static_cast<const T*>(L.x_t), L.dt_t, L.A,
                              static_cast<const T*>(L.B_t), static_cast<const T*>(L.C_t), L.D,
                              static_cast<T*>(L.y_t), blockIdx.x, nheads, headdim, ngroups, dstate);
}

// ---------------------------------------------------------------- several steps, one launch
// `steps` successive tokens of one layer in one launch (the device-side counterpart of a
// generation loop that advances the cache with no host round trip per token, when the
// tokens' inputs are on the device already).  One CTA per (b, h) keeps that unit's state in
// registers for all the steps, so the state is read once and written once.
//
// Lanes: the 4 lanes of a group share R rows of the state (group j of warp w holds rows
// w 8R + j + 8i, i < R), and lane L of the group the quads q = L + 4m (m < 8) of each row.
// A row's output is then summed in the single step's order without most of its shuffles:
// the single step forms one partial per quad (4 FMAs in order) and folds the 32 partials by
// the xor tree 16, 8, 4, 2, 1 over the quad index; here the levels 16, 8 and 4 pair quads of
// the same lane (m ^ 4, m ^ 2, m ^ 1) and only the levels 2 and 1 cross lanes.  Every level
// adds the same two partials, so the results equal `steps` launches of decode_step_kernel
// bit for bit (absent quads, dstate < 128, add the same +0 partials there and here).
//
// Inputs: the steps' x, B_t and C_t rows stream through a ring of kStepStages shared-memory
// stages filled kStepAhead steps ahead -- step j by lane 0 of warp j % 8, so the issuing is
// spread over the warps and stage w is always filled by warp w -- the rows by bulk copies (headdim and
// dstate are multiples of 8 and the pointers 16-byte aligned, so every row copy is 16-byte
// aligned and sized) and dt by a 4-byte cp.async that the stage's barrier also waits for.  A
// warp releases a stage after its step's arithmetic, so B_t and C_t are read from shared
// memory where they are used.  Inputs and outputs are [steps][...] arrays of the single
// step's layouts.  Every wait is bounded: expiry records SSD_ERR_TIMEOUT, the CTA stops
// stepping, waits for its copies in flight and writes back the state it has.
constexpr int kStepStages = 8;
constexpr int kStepAhead = 6;                          // the refilled stage was used 2 steps ago
static_assert(kStepStages == kDecodeWarps, "stage w is filled by warp w");

template <typename T>
__host__ __device__ constexpr int step_row_bytes(int n) { return (int)((n * sizeof(T) + 15) & ~size_t(15)); }

// The steps of U consecutive (b, h) units of one layer from `unit0` on (the CTA's whole
// work).  U = 2 takes two heads of one batch row and one group (they share B_t and C_t): row
// i of a lane group then belongs to unit i / R, so each warp carries two independent chains.
// FULL: dstate is 128, so every lane holds all 8 of its quads (no per-quad presence tests).
template <typename T, int R, int U, bool FULL>
__device__ __forceinline__ void steps_unit(float* __restrict__ state, const T* __restrict__ x,
                                           const float* __restrict__ dt, const float* __restrict__ A,
                                           const T* __restrict__ Bm, const T* __restrict__ Cm,
                                           const float* __restrict__ D, T* __restrict__ y, int steps, int batch,
                                           int nheads, int headdim, int ngroups, int dstate, int unit0, int* err)
{
    static_assert(R == 1 || R == 2, "rows per lane group");
    static_assert(U == 1 || (U == 2 && R == 1), "units per CTA");
    constexpr int NR = R * U;                          // rows per lane
    // per stage: the units' x rows | B_t row | C_t row | the units' dt
    extern __shared__ __align__(16) uint8_t stage_mem[];
    __shared__ __align__(8) uint64_t full[kStepStages], empty[kStepStages];
    __shared__ int abort_flag;
    const int xbytes = step_row_bytes<T>(U * headdim);
    const int nbytes = step_row_bytes<T>(dstate);
    const int stage_bytes = xbytes + 2 * nbytes + 16;

    const int b = unit0 / nheads;
    const int h0 = unit0 - b * nheads;
    const int g = h0 / (nheads / ngroups);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int grp = lane >> 2, L = lane & 3;
    const int nq = FULL ? 32 : dstate >> 2;            // quads in a row (<= 32)
    const int p0 = warp * 8 * R;                       // row of lane row i: p0 + 8 (i % R) + grp
    const size_t units = (size_t)batch * nheads;
    float Ah[U], Dh[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        Ah[u] = A[h0 + u];
        Dh[u] = D[h0 + u];
    }
    volatile int* abort = &abort_flag;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStepStages; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], kDecodeWarps);
        }
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();

    // lane 0 of warp k % kStepStages: the copies of step k into stage k % kStepStages, once
    // every warp has finished the step that used the stage before
    int last_issued = -1;
    auto issue = [&](int k) -> bool {
        const int st = k % kStepStages;
        if (k >= kStepStages && !ptx::mbar_wait_or_abort(&empty[st], ((k / kStepStages) - 1) & 1, err, abort))
            return false;
        uint8_t* sp = stage_mem + (size_t)st * stage_bytes;
        const size_t bc = ((size_t)k * batch * ngroups + (size_t)b * ngroups + g) * dstate;
        if (U == 1)
            ptx::cp_async_4(sp + xbytes + 2 * nbytes, dt + (size_t)k * units + unit0);
        else
            ptx::cp_async_8(sp + xbytes + 2 * nbytes, dt + (size_t)k * units + unit0);
        ptx::cp_async_mbar_arrive(&full[st]);          // before the arrival below
        ptx::mbar_expect_tx(&full[st], (uint32_t)((U * headdim + 2 * dstate) * sizeof(T)));
        ptx::bulk_load(sp, x + ((size_t)k * units + unit0) * headdim, U * headdim * sizeof(T), &full[st]);
        ptx::bulk_load(sp + xbytes, Bm + bc, dstate * sizeof(T), &full[st]);
        ptx::bulk_load(sp + xbytes + nbytes, Cm + bc, dstate * sizeof(T), &full[st]);
        last_issued = k;
        return true;
    };
    if (lane == 0 && warp < steps && warp < kStepAhead) issue(warp);

    // rows of this lane that exist (headdim is a multiple of 8: all 8 groups of a warp agree)
    bool row_on[NR];
    float* S[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const int p = p0 + 8 * (i % R) + grp;
        row_on[i] = p0 + 8 * (i % R) < headdim;
        S[i] = state + ((size_t)(unit0 + i / R) * headdim + p) * dstate;
    }
    float4 s[NR][8];
#pragma unroll
    for (int i = 0; i < NR; ++i)
#pragma unroll
        for (int m = 0; m < 8; ++m)
            s[i][m] = row_on[i] && L + 4 * m < nq ? *reinterpret_cast<const float4*>(S[i] + 4 * (L + 4 * m))
                                                  : make_float4(0.f, 0.f, 0.f, 0.f);

    for (int k = 0; k < steps; ++k) {
        if (lane == 0 && k + kStepAhead < steps && (k + kStepAhead) % kStepStages == warp && !issue(k + kStepAhead))
            *abort = 1;
        const int st = k % kStepStages;
        if (!ptx::mbar_wait_or_abort(&full[st], (k / kStepStages) & 1, err, abort)) break;
        const uint8_t* sp = stage_mem + (size_t)st * stage_bytes;
        const T* sx = reinterpret_cast<const T*>(sp);
        const T* sb = reinterpret_cast<const T*>(sp + xbytes);
        const T* sc = reinterpret_cast<const T*>(sp + xbytes + nbytes);
        float dtv[U], a[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            dtv[u] = reinterpret_cast<const float*>(sp + xbytes + 2 * nbytes)[u];
            a[u] = expf(dtv[u] * Ah[u]);               // fp32 decay exponent
        }
        float xv[NR], acc[NR];
#pragma unroll
        for (int i = 0; i < NR; ++i)
            xv[i] = row_on[i] ? Elem<T>::load(sx + (i / R) * headdim + p0 + 8 * (i % R) + grp) : 0.f;
        float part[NR][8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const bool qon = L + 4 * m < nq;
            const float4 bq = qon ? load4<T>(sb + 4 * (L + 4 * m)) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 cq = qon ? load4<T>(sc + 4 * (L + 4 * m)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < NR; ++i) {
                const float dx = dtv[i / R] * xv[i];
                float pa = 0.f;
                if (qon) {
                    // a v + (dx b) per element, two elements per packed instruction
                    const float2 dx2 = make_float2(dx, dx), a2 = make_float2(a[i / R], a[i / R]);
                    float4 v = s[i][m];
                    const float2 vxy = ptx::ffma2(a2, make_float2(v.x, v.y), ptx::fmul2(dx2, make_float2(bq.x, bq.y)));
                    const float2 vzw = ptx::ffma2(a2, make_float2(v.z, v.w), ptx::fmul2(dx2, make_float2(bq.z, bq.w)));
                    v = make_float4(vxy.x, vxy.y, vzw.x, vzw.y);
                    pa = fmaf(cq.x, v.x, pa);
                    pa = fmaf(cq.y, v.y, pa);
                    pa = fmaf(cq.z, v.z, pa);
                    pa = fmaf(cq.w, v.w, pa);
                    s[i][m] = v;
                }
                part[i][m] = pa;
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[st]);   // the stage may be refilled
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            // quad levels 16, 8, 4 inside the lane, then 2 and 1 across the group
            float t0 = part[i][0] + part[i][4], t1 = part[i][1] + part[i][5];
            float t2 = part[i][2] + part[i][6], t3 = part[i][3] + part[i][7];
            t0 = t0 + t2;
            t1 = t1 + t3;
            float v = t0 + t1;
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            acc[i] = v;
        }
        if (L == 0) {
#pragma unroll
            for (int i = 0; i < NR; ++i)
                if (row_on[i])
                    Elem<T>::store(y + ((size_t)k * units + unit0 + i / R) * headdim + p0 + 8 * (i % R) + grp,
                                   fmaf(Dh[i / R], xv[i], acc[i]));
        }
        if (*abort) break;
    }
#pragma unroll
    for (int i = 0; i < NR; ++i)
#pragma unroll
        for (int m = 0; m < 8; ++m)
            if (row_on[i] && L + 4 * m < nq) *reinterpret_cast<float4*>(S[i] + 4 * (L + 4 * m)) = s[i][m];
    // the CTA does not exit with copies in flight: each warp waits for the last fill of its stage
    __syncthreads();
    if (lane == 0 && last_issued >= 0)
        ptx::mbar_wait(&full[last_issued % kStepStages], (last_issued / kStepStages) & 1, err);
}

// CTAs an SM holds: three with one row per lane, two with two rows of two units, one with
// two rows of one unit (its register count is above 128)
template <int R, int U>
constexpr int steps_ctas_per_sm() { return R * U == 1 ? 3 : (R == 1 ? 2 : 1); }

template <typename T, int R, int U, bool FULL>
__global__ void __launch_bounds__(kDecodeThreads, steps_ctas_per_sm<R, U>())
decode_steps_kernel(float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
                    const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
                    const float* __restrict__ D, T* __restrict__ y, int steps, int batch, int nheads,
                    int headdim, int ngroups, int dstate, int* err)
{
    steps_unit<T, R, U, FULL>(state, x, dt, A, Bm, Cm, D, y, steps, batch, nheads, headdim, ngroups, dstate,
                              blockIdx.x * U, err);
}

// The same for every layer of a table (blockIdx.y = layer): each entry's per-step pointers
// address [steps][...] arrays, so one launch advances the whole stack by `steps` tokens.
template <typename T, int R, int U, bool FULL>
__global__ void __launch_bounds__(kDecodeThreads, steps_ctas_per_sm<R, U>())
decode_steps_layers_kernel(const ssd_decode_layer_t* __restrict__ layers, int steps, int batch, int nheads,
                           int headdim, int ngroups, int dstate, int* err)
{
    const ssd_decode_layer_t L = layers[blockIdx.y];
    if (!layer_entry_ok(L, err)) return;
    steps_unit<T, R, U, FULL>(L.state, static_cast<const T*>(L.x_t), L.dt_t, L.A, static_cast<const T*>(L.B_t),
                              static_cast<const T*>(L.C_t), L.D, static_cast<T*>(L.y_t), steps, batch, nheads,
                              headdim, ngroups, dstate, blockIdx.x * U, err);
}

// Shapes whose state does not fit in registers: the single step's body once per step, still
// one launch (each CTA owns its unit's state, so the steps need no synchronisation).
template <typename T, int QPL, int ROWS>
__device__ __forceinline__ void steps_loop_unit(float* __restrict__ state, const T* __restrict__ x,
                                                const float* __restrict__ dt, const float* __restrict__ A,
                                                const T* __restrict__ Bm, const T* __restrict__ Cm,
                                                const float* __restrict__ D, T* __restrict__ y, int steps,
                                                int batch, int nheads, int headdim, int ngroups, int dstate)
{
    const size_t units = (size_t)batch * nheads;
    for (int k = 0; k < steps; ++k)
        decode_unit<T, QPL, ROWS>(state, x + (size_t)k * units * headdim, dt + (size_t)k * units, A,
                                  Bm + (size_t)k * batch * ngroups * dstate, Cm + (size_t)k * batch * ngroups * dstate,
                                  D, y + (size_t)k * units * headdim, blockIdx.x, nheads, headdim, ngroups, dstate);
}

template <typename T, int QPL, int ROWS>
__global__ void __launch_bounds__(kDecodeThreads, QPL == 1 ? 4 : 2)
decode_steps_loop_kernel(float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
                         const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
                         const float* __restrict__ D, T* __restrict__ y, int steps, int batch, int nheads,
                         int headdim, int ngroups, int dstate)
{
    steps_loop_unit<T, QPL, ROWS>(state, x, dt, A, Bm, Cm, D, y, steps, batch, nheads, headdim, ngroups, dstate);
}

template <typename T, int QPL, int ROWS>
__global__ void __launch_bounds__(kDecodeThreads, QPL == 1 ? 4 : 2)
decode_steps_layers_loop_kernel(const ssd_decode_layer_t* __restrict__ layers, int steps, int batch,
                                int nheads, int headdim, int ngroups, int dstate, int* err)
{
    const ssd_decode_layer_t L = layers[blockIdx.y];
    if (!layer_entry_ok(L, err)) return;
    steps_loop_unit<T, QPL, ROWS>(L.state, static_cast<const T*>(L.x_t), L.dt_t, L.A,
                                  static_cast<const T*>(L.B_t), static_cast<const T*>(L.C_t), L.D,
                                  static_cast<T*>(L.y_t), steps, batch, nheads, headdim, ngroups, dstate);
}

// Two units per CTA where a pair of heads shares B_t and C_t, every quad is present, and the
// units (of all layers) are more than one wave of one-unit CTAs: below that, one unit a CTA
// keeps more SMs busy (a batch-1 layer has 80 units for 148 SMs).
bool steps_pair(const Dims& d, int n_layers)
{
    const long long units = (long long)d.batch * d.nheads * n_layers;
    return d.dstate == 128 && d.headdim <= 64 && (d.nheads / d.ngroups) % 2 == 0 &&
           units > (long long)steps_ctas_per_sm<1, 1>() * tc_sm_count();
}

// Dynamic shared memory of the multi-step kernels: the ring of input stages.
template <typename T>
size_t steps_smem(const Dims& d, int units_per_cta)
{
    return (size_t)kStepStages *
           (step_row_bytes<T>(units_per_cta * d.headdim) + 2 * step_row_bytes<T>(d.dstate) + 16);
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
    int* err = device_error_word();
    const bool full = d.dstate == 128;
    if (steps_pair(d, 1)) {
        decode_steps_kernel<T, 1, 2, true><<<grid / 2, kDecodeThreads, steps_smem<T>(d, 2), s>>>(
            state, xt, dt, A, Bt, Ct, D, yt, steps, d.batch, d.nheads, d.headdim, d.ngroups, d.dstate, err);
    } else if (d.dstate <= 128 && d.headdim <= 64) {
        auto k = full ? decode_steps_kernel<T, 1, 1, true> : decode_steps_kernel<T, 1, 1, false>;
        k<<<grid, kDecodeThreads, steps_smem<T>(d, 1), s>>>(state, xt, dt, A, Bt, Ct, D, yt, steps, d.batch,
                                                            d.nheads, d.headdim, d.ngroups, d.dstate, err);
    } else if (d.dstate <= 128) {
        auto k = full ? decode_steps_kernel<T, 2, 1, true> : decode_steps_kernel<T, 2, 1, false>;
        k<<<grid, kDecodeThreads, steps_smem<T>(d, 1), s>>>(state, xt, dt, A, Bt, Ct, D, yt, steps, d.batch,
                                                            d.nheads, d.headdim, d.ngroups, d.dstate, err);
    } else if (d.dstate <= 256) {
        decode_steps_loop_kernel<T, 2, 4><<<grid, kDecodeThreads, 0, s>>>(state, xt, dt, A, Bt, Ct, D, yt, steps,
                                                                          d.batch, d.nheads, d.headdim, d.ngroups,
                                                                          d.dstate);
    } else {
        decode_steps_loop_kernel<T, 4, 2><<<grid, kDecodeThreads, 0, s>>>(state, xt, dt, A, Bt, Ct, D, yt, steps,
                                                                          d.batch, d.nheads, d.headdim, d.ngroups,
                                                                          d.dstate);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_steps_layers_dtype(const Dims& d, const ssd_decode_layer_t* layers, int n_layers, int steps,
                                      cudaStream_t s)
{
    const dim3 grid((unsigned)(d.batch * d.nheads), (unsigned)n_layers);
    int* err = device_error_word();
    const bool full = d.dstate == 128;
    if (steps_pair(d, n_layers)) {
        decode_steps_layers_kernel<T, 1, 2, true><<<dim3(grid.x / 2, grid.y), kDecodeThreads, steps_smem<T>(d, 2), s>>>(
            layers, steps, d.batch, d.nheads, d.headdim, d.ngroups, d.dstate, err);
    } else if (d.dstate <= 128 && d.headdim <= 64) {
        auto k = full ? decode_steps_layers_kernel<T, 1, 1, true> : decode_steps_layers_kernel<T, 1, 1, false>;
        k<<<grid, kDecodeThreads, steps_smem<T>(d, 1), s>>>(layers, steps, d.batch, d.nheads, d.headdim, d.ngroups,
                                                            d.dstate, err);
    } else if (d.dstate <= 128) {
        auto k = full ? decode_steps_layers_kernel<T, 2, 1, true> : decode_steps_layers_kernel<T, 2, 1, false>;
        k<<<grid, kDecodeThreads, steps_smem<T>(d, 1), s>>>(layers, steps, d.batch, d.nheads, d.headdim, d.ngroups,
                                                            d.dstate, err);
    } else if (d.dstate <= 256) {
        decode_steps_layers_loop_kernel<T, 2, 4><<<grid, kDecodeThreads, 0, s>>>(layers, steps, d.batch, d.nheads,
                                                                                 d.headdim, d.ngroups, d.dstate, err);
    } else {
        decode_steps_layers_loop_kernel<T, 4, 2><<<grid, kDecodeThreads, 0, s>>>(layers, steps, d.batch, d.nheads,
                                                                                 d.headdim, d.ngroups, d.dstate, err);
    }
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

cudaError_t launch_decode_steps_layers(const Dims& d, ssd_dtype_t dtype, const ssd_decode_layer_t* layers,
                                       int n_layers, int steps, cudaStream_t s)
{
    if (d.batch == 0 || n_layers == 0 || steps == 0) return cudaSuccess;
    if (dtype == SSD_F32) return launch_steps_layers_dtype<float>(d, layers, n_layers, steps, s);
    return launch_steps_layers_dtype<__nv_bfloat16>(d, layers, n_layers, steps, s);
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
