// Tensor-core stages of the bf16 chunked SSD prefill on sm_100a: tcgen05.mma with
// TMEM accumulators, operands staged in shared memory by TMA (128-byte swizzle).
//
// "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching
// for Inference", section "2. Metodologia": the SSD layer is dominated by matrix
// contractions (einsums) inside fixed-size chunks, masked by a static
// lower-triangular decay mask whose exponents are taken in fp32.  On B200 those
// contractions run on the 5th-generation tensor cores (bf16 in, fp32 accumulate):
//
//   chunk_state_tc  (per b, chunk c, head h):
//       S_c^T = B_c^T (w o X_c)            M = dstate 128, N = headdim 64, K = chunk
//       with w_s = exp(Lam_end - Lam_s) dt_s applied to the rows of X in shared memory;
//       both operands are fp16 (converted in shared memory) so that the carried and
//       final states see 2^-12 rather than 2^-9 relative rounding per term.
//   chunk_output_tc (per b, c, h and 128-token tile t of the chunk):
//       G  = C_t B_{s<=t}^T               M = 128 tokens, N = 128 or 256 sources, K = dstate
//       Yo = C_t H_c^T                    M = 128, N = headdim, K = dstate
//       P  = G o exp(Lam_t - Lam_s) o dt_s (s <= t), rounded to bf16 in shared memory
//       Yd = P X_{s<=t}                   M = 128, N = headdim, K = 128 or 256
//       y  = Yd + exp(Lam_t) Yo + D_h x_t  -> bf16
//
// One thread issues all TMA loads and MMAs of a CTA; every wait on an mbarrier is
// bounded and records SSD_ERR_TIMEOUT in the device error word on expiry.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "prefill_tc.h"
#include "ptx.cuh"

namespace ssd {

using namespace ptx;

namespace {

constexpr int kTcThreads = 128;
constexpr int kBox = 16384;                    // one TMA box: 128 rows x 128 bytes

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Byte offset of 16-byte chunk q of row r in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int r, int q) { return r * 128 + ((q ^ (r & 7)) << 4); }

// ---------------------------------------------------------------- chunk state
template <int Q>
struct StateSmem {
    static constexpr int kB = 0;                   // [2 n-halves][Q rows][128 B]
    static constexpr int kX = 2 * Q * 128;         // [Q rows][128 B]
    static constexpr int kW = kX + Q * 128;        // float[Q]
    static constexpr int kBar = kW + Q * 4;        // 2 x mbarrier
    static constexpr int kSlot = kBar + 16;        // TMEM address
    static constexpr int kBytes = kSlot + 16 + 1024;
};

template <int Q>
__global__ void __launch_bounds__(kTcThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                      const float* __restrict__ dt, const float* __restrict__ lam,
                      float* __restrict__ states, int seqlen, int nheads, int ngroups, int nchunks,
                      int* err)
{
    using L = StateSmem<Q>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint8_t* sB = sm + L::kB;
    uint8_t* sX = sm + L::kX;
    float* sw = reinterpret_cast<float*>(sm + L::kW);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint32_t* slot = reinterpret_cast<uint32_t*>(sm + L::kSlot);

    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (nheads / ngroups);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = c * Q;
    const int qlen = min(Q, seqlen - t0);

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(slot, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;

    if (tid == 0) {
        mbar_expect_tx(&bars[0], 3 * Q * 128);
#pragma unroll
        for (int rb = 0; rb < Q / 128; ++rb) {
            tma_load_3d(sB + rb * kBox, &tm_b, g * 128, t0 + rb * 128, b, &bars[0]);
            tma_load_3d(sB + Q * 128 + rb * kBox, &tm_b, g * 128 + 64, t0 + rb * 128, b, &bars[0]);
            tma_load_3d(sX + rb * kBox, &tm_x, h * 64, t0 + rb * 128, b, &bars[0]);
        }
    }
    const float* lamc = lam + (((size_t)b * nheads + h) * nchunks + c) * Q;
    const float lam_end = lamc[Q - 1];
    for (int s = tid; s < Q; s += kTcThreads)
        sw[s] = s < qlen ? expf(lam_end - lamc[s]) * dt[((size_t)b * seqlen + t0 + s) * nheads + h] : 0.f;
    __syncthreads();

    bool ok = mbar_wait(&bars[0], 0, err);
    if (ok) {
        // Operands go to the tensor cores as fp16 (3 more mantissa bits than bf16; every
        // bf16 input and every w x product of these workloads is far inside fp16 range).
        // X~ = w o X and B are converted in place; a row's 16-byte chunks all belong to it.
        for (int s = tid; s < Q; s += kTcThreads) {
            const float w = sw[s];
            uint4* row = reinterpret_cast<uint4*>(sX + s * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint4 u = row[q];
                u.x = pack_f16x2(bf16lo(u.x) * w, bf16hi(u.x) * w);
                u.y = pack_f16x2(bf16lo(u.y) * w, bf16hi(u.y) * w);
                u.z = pack_f16x2(bf16lo(u.z) * w, bf16hi(u.z) * w);
                u.w = pack_f16x2(bf16lo(u.w) * w, bf16hi(u.w) * w);
                row[q] = u;
            }
        }
        for (int i = tid; i < 2 * Q * 8; i += kTcThreads) {
            uint4* chunk = reinterpret_cast<uint4*>(sB) + i;
            uint4 u = *chunk;
            u.x = pack_f16x2(bf16lo(u.x), bf16hi(u.x));
            u.y = pack_f16x2(bf16lo(u.y), bf16hi(u.y));
            u.z = pack_f16x2(bf16lo(u.z), bf16hi(u.z));
            u.w = pack_f16x2(bf16lo(u.w), bf16hi(u.w));
            *chunk = u;
        }
    }
    fence_proxy_async_smem();
    ok = __syncthreads_and(ok);

    if (tid == 0 && ok) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_f16_f32(128, 64, true, true);
        const uint32_t aB = smem_u32(sB), aX = smem_u32(sX);
#pragma unroll
        for (int ks = 0; ks < Q / 16; ++ks) {
            const uint64_t ad = smem_desc_sw128(aB + ks * 2048, Q * 128, 1024);
            const uint64_t bd = smem_desc_sw128(aX + ks * 2048, Q * 128, 1024);
            umma_bf16(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars[1]);
    }
    if (ok) ok = mbar_wait(&bars[1], 0, err);
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (ok) {
        uint32_t v0[32], v1[32];
        const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16);
        tmem_ld32(ta, v0);
        tmem_ld32(ta + 32, v1);
        tmem_wait_ld();
        const int n = warp * 32 + lane;
        float* out = states + (((size_t)b * nheads + h) * nchunks + c) * (64 * 128) + n;
#pragma unroll
        for (int p = 0; p < 32; ++p) out[p * 128] = __uint_as_float(v0[p]);
#pragma unroll
        for (int p = 0; p < 32; ++p) out[(p + 32) * 128] = __uint_as_float(v1[p]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

// ---------------------------------------------------------------- chunk output
template <int Q>
struct OutSmem {
    static constexpr int kC = 0;                        // [2 n-halves][128 rows][128 B]
    static constexpr int kB = 2 * kBox;                 // [2 n-halves][Q rows][128 B]
    static constexpr int kX = kB + 2 * Q * 128;         // [Q rows][128 B]
    static constexpr int kP = kX + Q * 128;             // [Q/64 s-blocks][128 rows][128 B]
    static constexpr int kH = kP + (Q / 64) * kBox;     // [2 n-halves][64 rows][128 B]
    static constexpr int kLam = kH + 2 * 8192;          // float[Q]
    static constexpr int kDt = kLam + Q * 4;            // float[Q]
    static constexpr int kBar = kDt + Q * 4;
    static constexpr int kSlot = kBar + 16;
    static constexpr int kBytes = kSlot + 16 + 1024;
};

constexpr uint32_t kColS = 0, kColYd = 256, kColYo = 320;

template <int Q>
__global__ void __launch_bounds__(kTcThreads, 1)
chunk_output_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_c, const float* __restrict__ dt,
                       const float* __restrict__ D, const float* __restrict__ lam,
                       const float* __restrict__ states, __nv_bfloat16* __restrict__ y, int seqlen,
                       int nheads, int ngroups, int nchunks, int* err)
{
    using L = OutSmem<Q>;
    constexpr int NT = Q / 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint8_t* sC = sm + L::kC;
    uint8_t* sB = sm + L::kB;
    uint8_t* sX = sm + L::kX;
    uint8_t* sP = sm + L::kP;
    uint8_t* sH = sm + L::kH;
    float* sLam = reinterpret_cast<float*>(sm + L::kLam);
    float* sDt = reinterpret_cast<float*>(sm + L::kDt);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint32_t* slot = reinterpret_cast<uint32_t*>(sm + L::kSlot);

    const int c = blockIdx.x / NT, it = blockIdx.x % NT, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (nheads / ngroups);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int R = 128 * (it + 1);                       // source tokens s in [0, R)
    const int t0 = c * Q;
    const int qlen = min(Q, seqlen - t0);

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;

    if (tid == 0) {
        mbar_expect_tx(&bars[0], 2 * kBox + (it + 1) * 3 * kBox);
        tma_load_3d(sC, &tm_c, g * 128, t0 + it * 128, b, &bars[0]);
        tma_load_3d(sC + kBox, &tm_c, g * 128 + 64, t0 + it * 128, b, &bars[0]);
        for (int rb = 0; rb <= it; ++rb) {
            tma_load_3d(sB + rb * kBox, &tm_b, g * 128, t0 + rb * 128, b, &bars[0]);
            tma_load_3d(sB + Q * 128 + rb * kBox, &tm_b, g * 128 + 64, t0 + rb * 128, b, &bars[0]);
            tma_load_3d(sX + rb * kBox, &tm_x, h * 64, t0 + rb * 128, b, &bars[0]);
        }
    }
    const float* lamc = lam + (((size_t)b * nheads + h) * nchunks + c) * Q;
    for (int s = tid; s < R; s += kTcThreads) {
        sLam[s] = lamc[s];
        sDt[s] = s < qlen ? dt[((size_t)b * seqlen + t0 + s) * nheads + h] : 0.f;
    }
    // carried state H_c [64][128] fp32 -> bf16, K-major swizzled B operand
    const float* Hc = states + (((size_t)b * nheads + h) * nchunks + c) * (64 * 128);
    for (int id = tid; id < 64 * 16; id += kTcThreads) {
        const int p = id >> 4, kb = (id >> 3) & 1, q = id & 7;
        const float4* src = reinterpret_cast<const float4*>(Hc + p * 128 + kb * 64 + q * 8);
        const float4 f0 = src[0], f1 = src[1];
        uint4 u;
        u.x = pack_bf16x2(f0.x, f0.y);
        u.y = pack_bf16x2(f0.z, f0.w);
        u.z = pack_bf16x2(f1.x, f1.y);
        u.w = pack_bf16x2(f1.z, f1.w);
        *reinterpret_cast<uint4*>(sH + kb * 8192 + sw128(p, q)) = u;
    }
    fence_proxy_async_smem();
    __syncthreads();

    bool ok = mbar_wait(&bars[0], 0, err);
    ok = __syncthreads_and(ok);
    if (tid == 0 && ok) {
        tc_fence_after();
        const uint32_t idS = idesc_bf16_f32(128, R, false, false);
        constexpr uint32_t idY = idesc_bf16_f32(128, 64, false, false);
        const uint32_t aC = smem_u32(sC), aB = smem_u32(sB), aH = smem_u32(sH);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t kb = ks >> 2, off = (ks & 3) * 32;
            const uint64_t ad = smem_desc_sw128(aC + kb * kBox + off, 16, 1024);
            const uint64_t bd = smem_desc_sw128(aB + kb * (Q * 128) + off, 16, 1024);
            umma_bf16(tmem + kColS, ad, bd, idS, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t kb = ks >> 2, off = (ks & 3) * 32;
            const uint64_t ad = smem_desc_sw128(aC + kb * kBox + off, 16, 1024);
            const uint64_t bd = smem_desc_sw128(aH + kb * 8192 + off, 16, 1024);
            umma_bf16(tmem + kColYo, ad, bd, idY, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars[1]);
    }
    if (ok) ok = mbar_wait(&bars[1], 0, err);
    ok = __syncthreads_and(ok);
    tc_fence_after();

    const int r = warp * 32 + lane;                     // TMEM lane = tile row
    const int tl = it * 128 + r;                        // token index within the chunk
    const float lam_t = sLam[tl];
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    if (ok) {
        for (int cb = 0; cb < R / 32; ++cb) {
            uint32_t v[32];
            tmem_ld32(trow + kColS + cb * 32, v);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int s0 = cb * 32 + 2 * j;
                const float p0 = s0 <= tl ? __uint_as_float(v[2 * j]) * expf(lam_t - sLam[s0]) * sDt[s0] : 0.f;
                const float p1 = s0 + 1 <= tl ? __uint_as_float(v[2 * j + 1]) * expf(lam_t - sLam[s0 + 1]) * sDt[s0 + 1] : 0.f;
                pk[j] = pack_bf16x2(p0, p1);
            }
            uint8_t* blk = sP + (cb >> 1) * kBox;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int q = (cb & 1) * 4 + k;
                *reinterpret_cast<uint4*>(blk + sw128(r, q)) =
                    make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && ok) {
        tc_fence_after();
        constexpr uint32_t idY = idesc_bf16_f32(128, 64, false, true);
        const uint32_t aP = smem_u32(sP), aX = smem_u32(sX);
        for (int ks = 0; ks < R / 16; ++ks) {
            const uint64_t ad = smem_desc_sw128(aP + (ks >> 2) * kBox + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(aX + ks * 2048, Q * 128, 1024);
            umma_bf16(tmem + kColYd, ad, bd, idY, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars[1]);
    }
    if (ok) ok = mbar_wait(&bars[1], 1, err);
    ok = __syncthreads_and(ok);
    tc_fence_after();

    if (ok) {
        const int tg = t0 + tl;
        const float e = expf(lam_t);
        const float Dh = D[h];
        const uint8_t* xrow = sX + tl * 128;
        __nv_bfloat16* yrow = y + (((size_t)b * seqlen + tg) * nheads + h) * 64;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t yd[32], yo[32];
            tmem_ld32(trow + kColYd + half * 32, yd);
            tmem_ld32(trow + kColYo + half * 32, yo);
            tmem_wait_ld();
            if (tl < qlen) {
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int q = half * 4 + qq;
                    const uint4 xu = *reinterpret_cast<const uint4*>(xrow + ((q ^ (tl & 7)) << 4));
                    const uint32_t xw[4] = {xu.x, xu.y, xu.z, xu.w};
                    uint32_t o[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int j = qq * 8 + 2 * k;
                        const float a0 = __uint_as_float(yd[j]) + e * __uint_as_float(yo[j]) + Dh * bf16lo(xw[k]);
                        const float a1 = __uint_as_float(yd[j + 1]) + e * __uint_as_float(yo[j + 1]) + Dh * bf16hi(xw[k]);
                        o[k] = pack_bf16x2(a0, a1);
                    }
                    *reinterpret_cast<uint4*>(yrow + q * 8) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// bf16 tensor [outer][rows][inner] read in boxes of 64 (inner) x 128 (rows), 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, rows, outer};
    cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int Q>
cudaError_t chunk_state_tc_t(const Dims& d, const CUtensorMap& mx, const CUtensorMap& mb,
                             const float* dt, const float* lam, float* states, cudaStream_t s)
{
    auto k = chunk_state_tc_kernel<Q>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         StateSmem<Q>::kBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(d.nchunks, d.nheads, d.batch);
    k<<<grid, kTcThreads, StateSmem<Q>::kBytes, s>>>(mx, mb, dt, lam, states, d.seqlen, d.nheads,
                                                     d.ngroups, d.nchunks, device_error_word());
    return cudaGetLastError();
}

template <int Q>
cudaError_t chunk_output_tc_t(const Dims& d, const CUtensorMap& mx, const CUtensorMap& mb,
                              const CUtensorMap& mc, const float* dt, const float* D,
                              const float* lam, const float* states, void* y, cudaStream_t s)
{
    auto k = chunk_output_tc_kernel<Q>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         OutSmem<Q>::kBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(d.nchunks * (Q / 128), d.nheads, d.batch);
    k<<<grid, kTcThreads, OutSmem<Q>::kBytes, s>>>(mx, mb, mc, dt, D, lam, states,
                                                   static_cast<__nv_bfloat16*>(y), d.seqlen,
                                                   d.nheads, d.ngroups, d.nchunks,
                                                   device_error_word());
    return cudaGetLastError();
}

}  // namespace

bool tc_prefill_supported(const Dims& d)
{
    return d.headdim == 64 && d.dstate == 128 && (d.chunk_len == 128 || d.chunk_len == 256);
}

cudaError_t launch_chunk_state_tc(const Dims& d, const void* x, const float* dt, const void* B,
                                  const float* lam, float* states, cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    CUtensorMap mx, mb;
    if (!make_map(&mx, x, (uint64_t)d.nheads * 64, d.seqlen, d.batch) ||
        !make_map(&mb, B, (uint64_t)d.ngroups * 128, d.seqlen, d.batch))
        return cudaErrorInvalidValue;
    if (d.chunk_len == 256) return chunk_state_tc_t<256>(d, mx, mb, dt, lam, states, s);
    return chunk_state_tc_t<128>(d, mx, mb, dt, lam, states, s);
}

cudaError_t launch_chunk_output_tc(const Dims& d, const void* x, const float* dt, const void* B,
                                   const void* C, const float* D, const float* lam,
                                   const float* states, void* y, cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    CUtensorMap mx, mb, mc;
    if (!make_map(&mx, x, (uint64_t)d.nheads * 64, d.seqlen, d.batch) ||
        !make_map(&mb, B, (uint64_t)d.ngroups * 128, d.seqlen, d.batch) ||
        !make_map(&mc, C, (uint64_t)d.ngroups * 128, d.seqlen, d.batch))
        return cudaErrorInvalidValue;
    if (d.chunk_len == 256) return chunk_output_tc_t<256>(d, mx, mb, mc, dt, D, lam, states, y, s);
    return chunk_output_tc_t<128>(d, mx, mb, mc, dt, D, lam, states, y, s);
}

}  // namespace ssd
