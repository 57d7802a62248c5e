// Chunked SSD prefill on the CUDA cores (fp32 arithmetic), plus the two kernels
// the tensor-core path shares with it: the per-chunk decay cumsum and the scan of
// chunk states across chunks.
//
// "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching
// for Inference", section "2. Metodologia": the recurrence splits into chunks of
// fixed size; inside a chunk it is a masked matrix product built from a static
// lower-triangular mask; across chunks only an N x P state per (batch, head) is
// carried; the decay exponents are formed in fp32 (here from a double-precision cumsum
// kept as two floats, so that differences stay exact).  For chunk c of head h with
// Lam_t the inclusive cumsum of dt*A over the chunk's tokens:
//   (1) Lam_t = sum_{r <= t, r in chunk} dt_r A_h
//   (2) y_t  = sum_{s <= t} (C_t . B_s) exp(Lam_t - Lam_s) dt_s x_s
//   (3) S_c  = sum_s exp(Lam_end - Lam_s) dt_s x_s B_s^T      (chunk state from zero)
//       H_{c+1} = exp(Lam_end) H_c + S_c                      (carried state)
//   (4) y_t += exp(Lam_t) H_c C_t + D_h x_t
// States are stored [headdim][dstate].  Tokens past seqlen in the last chunk act
// as dt = 0, x = 0 (an exact identity on the state).
#include "common.cuh"

namespace ssd {

namespace {

constexpr int kThreads = 256;

// ----------------------------------------------------------------------------------
// (1) per (b, chunk, head-tile): Lam over the chunk, written [b][h][c][2][Q] (hi, lo) for the
// CUDA-core path, or as the tensor-core path's decay factors.
// The chunk's dt block [Q][nheads] is contiguous in memory; it is staged through
// shared memory, transposed to [head][Q + 4], so that the global read is coalesced and
// both shared-memory sides are free of bank conflicts.
// ----------------------------------------------------------------------------------
constexpr int kCumsumHeads = 8;      // one warp per head
constexpr int kFacQ = 128;           // block length of the tensor-core path (decay factors)
static_assert(kMaxChunk * kCumsumHeads % kThreads == 0, "dt rows per thread");

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t u) {
    const float lo = __uint_as_float(u << 16), hi = __uint_as_float(u & 0xFFFF0000u);
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// exp(ref - Lambda_s) dt_s for four consecutive tokens
__device__ __forceinline__ float4 decay_times_dt(float ref, float4 lam, float4 dt)
{
    return make_float4(expf(ref - lam.x) * dt.x, expf(ref - lam.y) * dt.y, expf(ref - lam.z) * dt.z,
                       expf(ref - lam.w) * dt.w);
}

// Per (b, h, chunk) row of `fac` (stride fac_stride floats): without `extras`, Lam summed in
// double as hi[Q] and lo[Q] floats; with `extras` (Q = kFacQ), Lam[Q] in fp32 and also
// dt[Q] (zero past seqlen) and the column factors of each 32-token sub-block,
// exp(Lam_last - Lam_s) dt_s and exp(Lam_first - Lam_s) dt_s.  With `wts`, the chunk-state
// weights exp(Lam_end - Lam_s) dt_s, exp(Lam_end) and three zeros ([b][h][c][Q + 4]); with
// `b_f16`, an fp16 copy of B.  Six CTAs fit on an SM (at most 42 registers a thread): on long
// prefills the grid is several waves of short CTAs, each a chain of memory round trips.
__global__ void __launch_bounds__(kThreads, 6)
chunk_cumsum_kernel(const float* __restrict__ dt, const float* __restrict__ A,
                    float* __restrict__ fac, int fac_stride, bool extras, float* __restrict__ wts,
                    const uint4* __restrict__ b_bf16, uint4* __restrict__ b_f16,
                    int b_row_chunks, int seqlen, int nheads, int Q, int nchunks,
                    const float* __restrict__ dt_bias, int dt_softplus, const int* __restrict__ vl_cu,
                    const int* __restrict__ vl_first, const int* __restrict__ vl_seq)
{
    extern __shared__ float sm_dt[];                   // [kCumsumHeads][Q + 4]
    // the next kernel of the stream (launched as a programmatic dependent) may stage its setup
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int c = blockIdx.x, h0 = blockIdx.y * kCumsumHeads, b = blockIdx.z;
    const int nh = min(kCumsumHeads, nheads - h0);
    // rows t0 .. t0 + valid - 1 of batch b are this chunk's tokens; in packed variable-length
    // mode (batch 1) chunk c is a block of one sequence, and rows past its end (the next
    // sequence's) count as padding: dt = 0
    int t0 = c * Q, valid = min(Q, seqlen - c * Q);
    if (vl_seq) {
        int sq;
        if (!varlen_block(vl_cu, vl_first, vl_seq, c, Q, &sq, &t0, &valid)) return;
    }
    // every dt load of this thread is issued before any is used, and the B copy's loads below
    // go out while they are in flight; the values land in shared memory after the copy
    constexpr int kDtPer = kMaxChunk * kCumsumHeads / kThreads;
    float raw[kDtPer];
    bool use[kDtPer];
#pragma unroll
    for (int m = 0; m < kDtPer; ++m) {
        const int i = threadIdx.x + m * kThreads;
        const int t = i / kCumsumHeads, hh = i - t * kCumsumHeads;
        use[m] = i < Q * kCumsumHeads && hh < nh && t < valid;
        raw[m] = use[m] ? dt[((size_t)b * seqlen + t0 + t) * nheads + h0 + hh] : 0.f;
    }
    if (b_f16) {
        // fp16 copy of this chunk's rows of B (bf16 -> fp16 is exact for these values'
        // range), the operand format of the tensor-core chunk-state GEMM; the head blocks
        // of a chunk split its rows between them
        const int rows = valid;
        const int r0 = (int)(((long long)rows * blockIdx.y) / gridDim.y);
        const int r1 = (int)(((long long)rows * (blockIdx.y + 1)) / gridDim.y);
        const size_t first = ((size_t)b * seqlen + (size_t)t0 + r0) * b_row_chunks;
        const int n = (r1 - r0) * b_row_chunks;
        constexpr int kUnroll = 4;
        for (int i0 = threadIdx.x; i0 < n; i0 += kUnroll * blockDim.x) {
            uint4 u[kUnroll];
#pragma unroll
            for (int j = 0; j < kUnroll; ++j) {
                const int i = i0 + j * blockDim.x;
                if (i < n) u[j] = b_bf16[first + i];
            }
#pragma unroll
            for (int j = 0; j < kUnroll; ++j) {
                const int i = i0 + j * blockDim.x;
                if (i < n) {
                    u[j].x = bf16x2_to_f16x2(u[j].x);
                    u[j].y = bf16x2_to_f16x2(u[j].y);
                    u[j].z = bf16x2_to_f16x2(u[j].z);
                    u[j].w = bf16x2_to_f16x2(u[j].w);
                    b_f16[first + i] = u[j];
                }
            }
        }
    }
    const int ldt = Q + 4;
#pragma unroll
    for (int m = 0; m < kDtPer; ++m) {
        const int i = threadIdx.x + m * kThreads;
        const int t = i / kCumsumHeads, hh = i - t * kCumsumHeads;
        if (i < Q * kCumsumHeads)
            sm_dt[hh * ldt + t] = use[m] ? dt_value(raw[m], dt_bias, dt_softplus, h0 + hh) : 0.f;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (!extras && warp < nh) {
        // CUDA-core path: Lambda summed in double and stored as two floats, hi = fl(Lambda) and
        // lo = fl(Lambda - hi), so that exp(Lam_t - Lam_s) stays exact to fp32 even where
        // |Lambda| is in the thousands (strong decay): [Q] hi, then [Q] lo
        const int hh = warp;
        const double Ah = A[h0 + hh];
        double carry = 0.0;
        float* f = fac + (((size_t)b * nheads + h0 + hh) * nchunks + c) * fac_stride;
        for (int j = 0; j * 32 < Q; ++j) {
            const int t = j * 32 + lane;
            double v = (t < Q) ? (double)sm_dt[hh * ldt + t] * Ah : 0.0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            v += carry;
            if (t < Q) {
                const float hi = (float)v;
                f[t] = hi;
                f[Q + t] = (float)(v - (double)hi);
            }
            carry = __shfl_sync(0xffffffffu, v, 31);
        }
        return;
    }
    if (warp < nh) {
        // tensor-core path (Q = kFacQ): lane l owns tokens 4l .. 4l + 3, so one warp scan covers
        // the block and each factor row goes out as one 16-byte store per lane
        const int hh = warp;
        const float Ah = A[h0 + hh];
        const float4 d = *reinterpret_cast<const float4*>(sm_dt + hh * ldt + 4 * lane);
        const float v0 = d.x * Ah, v1 = v0 + d.y * Ah, v2 = v1 + d.z * Ah, v3 = v2 + d.w * Ah;
        float tot = v3;                                  // inclusive scan of the lanes' sums
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, tot, o);
            if (lane >= o) tot += u;
        }
        float pre = __shfl_up_sync(0xffffffffu, tot, 1);
        if (lane == 0) pre = 0.f;
        const float4 v = make_float4(pre + v0, pre + v1, pre + v2, pre + v3);
        // Lambda at the block's last token, and at the last and first token of this lane's
        // 32-token sub-block (lanes 8j .. 8j + 7 hold sub-block j)
        const float lam_end = __shfl_sync(0xffffffffu, v.w, 31);
        const float lam_last = __shfl_sync(0xffffffffu, v.w, lane | 7);
        const float lam_first = __shfl_sync(0xffffffffu, v.x, lane & ~7);
        const size_t unit = ((size_t)b * nheads + h0 + hh) * nchunks + c;
        float4* f = reinterpret_cast<float4*>(fac + unit * fac_stride) + lane;
        f[0] = v;
        f[kFacQ / 4] = d;
        f[kFacQ / 2] = decay_times_dt(lam_last, v, d);
        f[3 * kFacQ / 4] = decay_times_dt(lam_first, v, d);
        if (wts) {
            // chunk-state weights w_s = exp(Lambda_end - Lambda_s) dt_s, then the block's decay
            // exp(Lambda_end) and zero padding: Q + 4 floats per row
            float4* wr = reinterpret_cast<float4*>(wts + unit * (kFacQ + 4));
            wr[lane] = decay_times_dt(lam_end, v, d);
            if (lane == 0) wr[kFacQ / 4] = make_float4(expf(lam_end), 0.f, 0.f, 0.f);
        }
    }
}

// ----------------------------------------------------------------------------------
// (3a) per (b, h, c): chunk state S_c[p][n] = sum_s w_s x_s[p] B_s[n],
//      w_s = exp(Lam_end - Lam_s) dt_s.
// Thread (ty, tx): tx owns the n-quad 4tx..4tx+3, ty owns rows ty + rpp*k.
// ----------------------------------------------------------------------------------
constexpr int kTokTile = 32;
constexpr int kMaxRows = 8;

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_state_simt_kernel(const T* __restrict__ x, const float* __restrict__ dt,
                        const T* __restrict__ Bm, const float* __restrict__ lam,
                        float* __restrict__ states, int seqlen, int nheads, int headdim,
                        int ngroups, int dstate, int Q, int nchunks, const float* __restrict__ dt_bias,
                        int dt_softplus, const int* __restrict__ vl_cu, const int* __restrict__ vl_first,
                        const int* __restrict__ vl_seq)
{
    extern __shared__ float sm[];
    float* sx = sm;                                    // [kTokTile][headdim]
    float* sb = sx + kTokTile * headdim;               // [kTokTile][dstate]
    float* sw = sb + kTokTile * dstate;                // [kTokTile]
    const int c = blockIdx.x, h = blockIdx.y;
    int b = blockIdx.z, t0 = c * Q, qlen = min(Q, seqlen - c * Q);
    if (vl_seq) {                                      // packed variable-length: chunk c of the table
        int sq;
        if (!varlen_block(vl_cu, vl_first, vl_seq, c, Q, &sq, &t0, &qlen)) return;
        b = 0;
    }
    const int g = h / (nheads / ngroups);
    const float* lamc = lam + (((size_t)b * nheads + h) * nchunks + c) * 2 * Q;   // hi, then lo
    const float* lamlo = lamc + Q;
    const float lam_end = lamc[Q - 1], lam_end_lo = lamlo[Q - 1];

    const int nq = dstate >> 2;
    const int rpp = kThreads / nq;                     // rows per pass
    const int tx = threadIdx.x % nq, ty = threadIdx.x / nq;
    const bool active = ty < rpp;
    float* out = states + (((size_t)b * nheads + h) * nchunks + c) * headdim * dstate;

    for (int pbase = 0; pbase < headdim; pbase += rpp * kMaxRows) {
        float4 acc[kMaxRows];
#pragma unroll
        for (int k = 0; k < kMaxRows; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < qlen; s0 += kTokTile) {
            const int ns = min(kTokTile, qlen - s0);
            __syncthreads();
            for (int i = threadIdx.x; i < kTokTile * headdim; i += kThreads) {
                const int s = i / headdim, p = i - s * headdim;
                sx[i] = s < ns ? Elem<T>::load(x + (((size_t)b * seqlen + t0 + s0 + s) * nheads + h) * headdim + p) : 0.f;
            }
            for (int i = threadIdx.x; i < kTokTile * dstate; i += kThreads) {
                const int s = i / dstate, n = i - s * dstate;
                sb[i] = s < ns ? Elem<T>::load(Bm + (((size_t)b * seqlen + t0 + s0 + s) * ngroups + g) * dstate + n) : 0.f;
            }
            if (threadIdx.x < kTokTile) {
                const int s = threadIdx.x;
                sw[s] = s < ns ? expf((lam_end - lamc[s0 + s]) + (lam_end_lo - lamlo[s0 + s])) *
                                     dt_value(dt[((size_t)b * seqlen + t0 + s0 + s) * nheads + h], dt_bias, dt_softplus, h)
                               : 0.f;
            }
            __syncthreads();
            if (active) {
                for (int s = 0; s < ns; ++s) {
                    const float4 bv = *reinterpret_cast<const float4*>(sb + s * dstate + 4 * tx);
                    const float ws = sw[s];
#pragma unroll
                    for (int k = 0; k < kMaxRows; ++k) {
                        const int p = pbase + ty + rpp * k;
                        if (p < headdim) {
                            const float xv = ws * sx[s * headdim + p];
                            acc[k].x = fmaf(xv, bv.x, acc[k].x);
                            acc[k].y = fmaf(xv, bv.y, acc[k].y);
                            acc[k].z = fmaf(xv, bv.z, acc[k].z);
                            acc[k].w = fmaf(xv, bv.w, acc[k].w);
                        }
                    }
                }
            }
        }
        if (active) {
#pragma unroll
            for (int k = 0; k < kMaxRows; ++k) {
                const int p = pbase + ty + rpp * k;
                if (p < headdim) *reinterpret_cast<float4*>(out + (size_t)p * dstate + 4 * tx) = acc[k];
            }
        }
    }
}

// ----------------------------------------------------------------------------------
// (3b) per (b, h): walk the chunks in order, replacing each chunk state S_c by the
// state at the chunk's start H_c, and write the final state.  Each thread owns four
// consecutive state elements.  In place: init_state may alias final_state.
// ----------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
state_scan_kernel(const float* __restrict__ lam, float* __restrict__ states,
                  const float* init_state, float* final_state, int nheads, int PN, int Q,
                  int nchunks, const int* __restrict__ vl_first)
{
    // chain bh = (b, h): chunks 0 .. nchunks - 1 of that row of the per-chunk arrays; in packed
    // variable-length mode bh = (sequence, h) and its chunks are the table's first[s] ..
    // first[s + 1] - 1 of row h (batch 1)
    const int bh = blockIdx.y;
    const int e = 4 * (blockIdx.x * kThreads + threadIdx.x);
    if (e >= PN) return;
    size_t row = (size_t)bh * nchunks;
    if (vl_first) {
        const int sq = bh / nheads, h = bh - sq * nheads;
        row = (size_t)h * nchunks + vl_first[sq];
        nchunks = vl_first[sq + 1] - vl_first[sq];
    }
    float4 hs = make_float4(0.f, 0.f, 0.f, 0.f);
    if (init_state) hs = *reinterpret_cast<const float4*>(init_state + (size_t)bh * PN + e);
    const float* lamr = lam + row * 2 * Q;             // per chunk: [Q] hi, then [Q] lo
    float* st = states + row * PN + e;
    float4 nxt = nchunks > 0 ? *reinterpret_cast<const float4*>(st) : hs;
    for (int c = 0; c < nchunks; ++c) {
        const float4 sc = nxt;
        if (c + 1 < nchunks) nxt = *reinterpret_cast<const float4*>(st + (size_t)(c + 1) * PN);
        *reinterpret_cast<float4*>(st + (size_t)c * PN) = hs;
        const float ec = expf(lamr[(size_t)c * 2 * Q + Q - 1]) * expf(lamr[(size_t)c * 2 * Q + 2 * Q - 1]);
        hs.x = fmaf(ec, hs.x, sc.x);
        hs.y = fmaf(ec, hs.y, sc.y);
        hs.z = fmaf(ec, hs.z, sc.z);
        hs.w = fmaf(ec, hs.w, sc.w);
    }
    *reinterpret_cast<float4*>(final_state + (size_t)bh * PN + e) = hs;
}

// ----------------------------------------------------------------------------------
// (2)+(4) per (b, h, c): y for the chunk's tokens, in tiles of kTokTile tokens.
//   y_t = sum_{s<=t} M[t][s] x_s + exp(Lam_t) H_c C_t + D x_t,
//   M[t][s] = (C_t . B_s) exp(Lam_t - Lam_s) dt_s.
// ----------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_output_simt_kernel(const T* __restrict__ x, const float* __restrict__ dt,
                         const T* __restrict__ Bm, const T* __restrict__ Cm,
                         const float* __restrict__ D, const float* __restrict__ lam,
                         const float* __restrict__ states, T* __restrict__ y, int seqlen,
                         int nheads, int headdim, int ngroups, int dstate, int Q, int nchunks,
                         const float* __restrict__ dt_bias, int dt_softplus, const int* __restrict__ vl_cu,
                         const int* __restrict__ vl_first, const int* __restrict__ vl_seq)
{
    extern __shared__ float sm[];
    float* sH = sm;                                    // [headdim][dstate + 1]
    const int ldH = dstate + 1;
    float* sC = sH + headdim * ldH;                    // [kTokTile][dstate + 1]
    float* sB = sC + kTokTile * ldH;                   // [kTokTile][dstate + 1]
    float* sX = sB + kTokTile * ldH;                   // [kTokTile][headdim]
    float* sM = sX + kTokTile * headdim;               // [kTokTile][kTokTile + 1]
    const int ldM = kTokTile + 1;
    float* sLs = sM + kTokTile * ldM;                  // [kTokTile] Lam_s
    float* sDs = sLs + kTokTile;                       // [kTokTile] dt_s
    float* sLl = sDs + kTokTile;                       // [kTokTile] low part of Lam_s

    const int c = blockIdx.x, h = blockIdx.y;
    int b = blockIdx.z, t0 = c * Q, qlen = min(Q, seqlen - c * Q);
    if (vl_seq) {                                      // packed variable-length: chunk c of the table
        int sq;
        if (!varlen_block(vl_cu, vl_first, vl_seq, c, Q, &sq, &t0, &qlen)) return;
        b = 0;
    }
    const int g = h / (nheads / ngroups);
    const float* lamc = lam + (((size_t)b * nheads + h) * nchunks + c) * 2 * Q;   // hi, then lo
    const float* lamlo = lamc + Q;
    const float* Hc = states + (((size_t)b * nheads + h) * nchunks + c) * headdim * dstate;
    const float Dh = D[h];
    const size_t tok_stride_x = (size_t)nheads * headdim;
    const size_t tok_stride_b = (size_t)ngroups * dstate;
    const T* xbase = x + ((size_t)b * seqlen + t0) * tok_stride_x + (size_t)h * headdim;
    T* ybase = y + ((size_t)b * seqlen + t0) * tok_stride_x + (size_t)h * headdim;
    const T* Bbase = Bm + ((size_t)b * seqlen + t0) * tok_stride_b + (size_t)g * dstate;
    const T* Cbase = Cm + ((size_t)b * seqlen + t0) * tok_stride_b + (size_t)g * dstate;

    for (int i = threadIdx.x; i < headdim * dstate; i += kThreads) {
        const int p = i / dstate, n = i - p * dstate;
        sH[p * ldH + n] = Hc[i];
    }

    // output tile: kTokTile x headdim, each thread owns (t = tid / tpr, p = tid % tpr + k*tpr)
    const int tpr = kThreads / kTokTile;               // threads per token row = 8
    const int my_t = threadIdx.x / tpr, my_p0 = threadIdx.x % tpr;

    for (int tt = 0; tt < qlen; tt += kTokTile) {
        const int nt = min(kTokTile, qlen - tt);
        __syncthreads();
        for (int i = threadIdx.x; i < kTokTile * dstate; i += kThreads) {
            const int t = i / dstate, n = i - t * dstate;
            sC[t * ldH + n] = t < nt ? Elem<T>::load(Cbase + (size_t)(tt + t) * tok_stride_b + n) : 0.f;
        }
        __syncthreads();
        // carried-state term and skip
        float acc[16];
        const int nper = (headdim + tpr - 1) / tpr;    // <= 16 for headdim <= 128
        const float lt = (my_t < nt) ? lamc[tt + my_t] : 0.f;
        const float et = (my_t < nt) ? expf(lt) * expf(lamlo[tt + my_t]) : expf(lt);
        for (int k = 0; k < nper; ++k) {
            const int p = my_p0 + k * tpr;
            float v = 0.f;
            if (p < headdim && my_t < nt) {
                const float* hr = sH + p * ldH;
                const float* cr = sC + my_t * ldH;
                for (int n = 0; n < dstate; ++n) v = fmaf(cr[n], hr[n], v);
                v *= et;
            }
            acc[k] = v;
        }
        // intra-chunk masked product, source tokens s <= t in tiles
        for (int ss = 0; ss <= tt; ss += kTokTile) {
            const int ns = min(kTokTile, qlen - ss);
            __syncthreads();
            for (int i = threadIdx.x; i < kTokTile * dstate; i += kThreads) {
                const int s = i / dstate, n = i - s * dstate;
                sB[s * ldH + n] = s < ns ? Elem<T>::load(Bbase + (size_t)(ss + s) * tok_stride_b + n) : 0.f;
            }
            for (int i = threadIdx.x; i < kTokTile * headdim; i += kThreads) {
                const int s = i / headdim, p = i - s * headdim;
                sX[i] = s < ns ? Elem<T>::load(xbase + (size_t)(ss + s) * tok_stride_x + p) : 0.f;
            }
            if (threadIdx.x < kTokTile) {
                const int s = threadIdx.x;
                sLs[s] = s < ns ? lamc[ss + s] : 0.f;
                sLl[s] = s < ns ? lamlo[ss + s] : 0.f;
                sDs[s] = s < ns ? dt_value(dt[((size_t)b * seqlen + t0 + ss + s) * nheads + h], dt_bias, dt_softplus, h)
                                : 0.f;
            }
            __syncthreads();
            // M tile: thread computes entries (t = i / kTokTile, s = i % kTokTile)
            for (int i = threadIdx.x; i < kTokTile * kTokTile; i += kThreads) {
                const int t = i / kTokTile, s = i - t * kTokTile;
                float m = 0.f;
                if (t < nt && s < ns && ss + s <= tt + t) {
                    const float* cr = sC + t * ldH;
                    const float* br = sB + s * ldH;
                    float cb = 0.f;
                    for (int n = 0; n < dstate; ++n) cb = fmaf(cr[n], br[n], cb);
                    m = cb * expf((lamc[tt + t] - sLs[s]) + (lamlo[tt + t] - sLl[s])) * sDs[s];
                }
                sM[t * ldM + s] = m;
            }
            __syncthreads();
            if (my_t < nt) {
                for (int k = 0; k < nper; ++k) {
                    const int p = my_p0 + k * tpr;
                    if (p < headdim) {
                        float v = acc[k];
                        for (int s = 0; s < ns; ++s) v = fmaf(sM[my_t * ldM + s], sX[s * headdim + p], v);
                        acc[k] = v;
                    }
                }
            }
        }
        if (my_t < nt) {
            const T* xr = xbase + (size_t)(tt + my_t) * tok_stride_x;
            T* yr = ybase + (size_t)(tt + my_t) * tok_stride_x;
            for (int k = 0; k < nper; ++k) {
                const int p = my_p0 + k * tpr;
                if (p < headdim) Elem<T>::store(yr + p, fmaf(Dh, Elem<T>::load(xr + p), acc[k]));
            }
        }
    }
}

// zero-length prefill: final = init (or zeros)
__global__ void copy_state_kernel(const float* init_state, float* final_state, size_t n)
{
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) final_state[i] = init_state ? init_state[i] : 0.f;
}

template <typename T>
cudaError_t chunk_state_simt_t(const Dims& d, const void* x, const float* dt, const void* B,
                               const float* lam, float* states, cudaStream_t s)
{
    const size_t smem = sizeof(float) * (kTokTile * (d.headdim + d.dstate) + kTokTile);
    auto k = chunk_state_simt_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(d.nchunks, d.nheads, d.batch);
    k<<<grid, kThreads, smem, s>>>(static_cast<const T*>(x), dt, static_cast<const T*>(B), lam,
                                   states, d.seqlen, d.nheads, d.headdim, d.ngroups, d.dstate,
                                   d.chunk_len, d.nchunks, d.dt_bias, d.dt_softplus, d.cu_seqlens, d.vl_first,
                                   d.vl_seq);
    return cudaGetLastError();
}

template <typename T>
cudaError_t chunk_output_simt_t(const Dims& d, const void* x, const float* dt, const void* B,
                                const void* C, const float* D, const float* lam,
                                const float* states, void* y, cudaStream_t s)
{
    const int ldH = d.dstate + 1;
    const size_t smem = sizeof(float) * ((size_t)d.headdim * ldH + 2 * kTokTile * ldH +
                                         kTokTile * d.headdim + kTokTile * (kTokTile + 1) +
                                         3 * kTokTile);
    auto k = chunk_output_simt_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(d.nchunks, d.nheads, d.batch);
    k<<<grid, kThreads, smem, s>>>(static_cast<const T*>(x), dt, static_cast<const T*>(B),
                                   static_cast<const T*>(C), D, lam, states, static_cast<T*>(y),
                                   d.seqlen, d.nheads, d.headdim, d.ngroups, d.dstate,
                                   d.chunk_len, d.nchunks, d.dt_bias, d.dt_softplus, d.cu_seqlens, d.vl_first,
                                   d.vl_seq);
    return cudaGetLastError();
}

}  // namespace

size_t simt_output_smem_bytes(int headdim, int dstate)
{
    const int ldH = dstate + 1;
    return sizeof(float) * ((size_t)headdim * ldH + 2 * kTokTile * ldH + kTokTile * headdim +
                            kTokTile * (kTokTile + 1) + 2 * kTokTile);
}

cudaError_t launch_chunk_cumsum(const Dims& d, const float* dt, const float* A, float* fac,
                                bool extras, float* wts, const void* b_bf16, void* b_f16,
                                cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    if (extras && d.chunk_len != kFacQ) return cudaErrorInvalidValue;
    const size_t smem = sizeof(float) * (d.chunk_len + 4) * kCumsumHeads;
    dim3 grid(d.nchunks, (d.nheads + kCumsumHeads - 1) / kCumsumHeads, d.batch);
    chunk_cumsum_kernel<<<grid, kThreads, smem, s>>>(
        dt, A, fac, extras ? 4 * d.chunk_len : 2 * d.chunk_len, extras, wts,
        static_cast<const uint4*>(b_bf16), static_cast<uint4*>(b_f16),
        d.ngroups * d.dstate / 8, d.seqlen, d.nheads, d.chunk_len, d.nchunks, d.dt_bias, d.dt_softplus,
        d.cu_seqlens, d.vl_first, d.vl_seq);
    return cudaGetLastError();
}

cudaError_t launch_chunk_state_simt(const Dims& d, ssd_dtype_t dtype, const void* x,
                                    const float* dt, const void* B, const float* lam,
                                    float* states, cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    if (dtype == SSD_F32) return chunk_state_simt_t<float>(d, x, dt, B, lam, states, s);
    return chunk_state_simt_t<__nv_bfloat16>(d, x, dt, B, lam, states, s);
}

cudaError_t launch_state_scan(const Dims& d, const float* lam, float* states,
                              const float* init_state, float* final_state, cudaStream_t s)
{
    if (d.batch == 0) return cudaSuccess;
    const int PN = d.headdim * d.dstate;
    dim3 grid((PN / 4 + kThreads - 1) / kThreads, (d.nseq ? d.nseq : d.batch) * d.nheads);
    state_scan_kernel<<<grid, kThreads, 0, s>>>(lam, states, init_state, final_state, d.nheads,
                                                PN, d.chunk_len, d.nchunks, d.vl_first);
    return cudaGetLastError();
}

cudaError_t launch_chunk_output_simt(const Dims& d, ssd_dtype_t dtype, const void* x,
                                     const float* dt, const void* B, const void* C,
                                     const float* D, const float* lam, const float* states,
                                     void* y, cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    if (dtype == SSD_F32) return chunk_output_simt_t<float>(d, x, dt, B, C, D, lam, states, y, s);
    return chunk_output_simt_t<__nv_bfloat16>(d, x, dt, B, C, D, lam, states, y, s);
}

cudaError_t launch_copy_state(const Dims& d, const float* init_state, float* final_state,
                              cudaStream_t s)
{
    const size_t n = (size_t)d.batch * d.nheads * d.headdim * d.dstate;
    if (n == 0) return cudaSuccess;
    copy_state_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(init_state, final_state, n);
    return cudaGetLastError();
}

}  // namespace ssd
