// Fused tensor-core prefill on sm_100a: one CTA walks the 128-token blocks of one to three
// heads of one (batch, group) in order, keeps their states in tensor memory and writes y,
// so that x is read once and no intermediate state goes through HBM.
//
// "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching for
// Inference", section "2. Metodologia": inside a chunk the SSD layer is a masked matrix
// contraction, and chunks talk only through the N x P state of each (batch, head).  With
// blocks of 128 tokens (a 256-token chunk is two blocks, its off-diagonal block entering
// through the state at the midpoint, an exact factorisation), t, s tokens of block k,
// Lam the inclusive cumsum of dt A from the block start and H_k the state at its start:
//
//   G_k   = C_k B_k^T                            (per (b, g, k): block_gram_kernel, bf16)
//   P     = G_k o exp(Lam_t - Lam_s) o dt_s       (s <= t), bf16, per head
//   y     = P X + exp(Lam_t) C_k H_k^T + D x      (bf16)
//   H_k+1 = exp(Lam_end) H_k + B_k^T (w o X),     w_s = exp(Lam_end - Lam_s) dt_s
//
// The state GEMM takes fp16 operands (B copied to fp16 by the cumsum kernel, exact for
// these values' range; w o X rounded to fp16): 3 more mantissa bits than bf16, which the
// state, summed over every block, needs.  G, P, X and the state image are bf16.
//
// chain_prefill_kernel, per CTA (b, g, heads hlo .. hlo + nh - 1), items i = k nh + j:
//   warp 0      TMA: C_k (staging), fp16 B_k (two-deep ring), x and the decay factors of each
//               item (four-deep ring of slots)
//   warp 1      tcgen05.mma, polling two streams: Yo_i = C H^T with C in TMEM and the state
//               image in shared memory, and S_i = B^T X~ accumulated onto the head's state in
//               TMEM; then Yd_i = P X with P in TMEM
//   warps 2-3   X~ = w o X (fp16) into a two-deep ring
//   warps 4-11  P from G_k (read from global memory a block ahead) and the decay factors
//   warps 12-15 the epilogue y = Yd + exp(Lam_t) Yo + D x, each warp TMA-storing its 32 rows
//   warps 16-19 the states: per item, the bf16 image of H for Yo, then H <- exp(Lam_end) H in
//               TMEM, onto which S accumulates
// Every wait is bounded; expiry records SSD_ERR_TIMEOUT in the device error word and the
// CTA drains without further waiting.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "prefill_tc.h"
#include "ptx.cuh"

namespace ssd {

using namespace ptx;

namespace {

constexpr int kBlk = 128;                       // tokens per block
constexpr int kP = 64, kN = 128;
constexpr int kBox = 16384;                     // one TMA box: 128 rows x 128 bytes
constexpr int kHImage = 16384;                  // bf16 state image: 2 x [128 n][32 p]
constexpr int kGramBytes = kBlk * kBlk * 2;     // bf16 G of one (b, g, block)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ================================================================ G = C B^T per block
// One CTA per (block k, group g, batch b): G_k = C_k B_k^T (K = N = 128) on the tensor
// cores, rounded to bf16 and stored as four planes of 32 columns, plane kc holding row t's
// columns 32 kc .. 32 kc + 31 as 64 contiguous bytes at t * 64 -- the order in which the
// chain kernel's P threads read them.
constexpr int kGramThreads = 128;

struct GramSmem {
    static constexpr int kC = 0;
    static constexpr int kB = 2 * kBox;
    static constexpr int kBar = 4 * kBox;
    static constexpr int kSlot = kBar + 16;
    static constexpr int kBytes = kSlot + 16 + 1024;
};

__global__ void __launch_bounds__(kGramThreads)
block_gram_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                  uint4* __restrict__ gram, int ngroups, int nblocks, int* err)
{
    using L = GramSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kSlot);
    griddep_launch_dependents();

    const int k = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    bool ok = true;
    if (tid == 0) {
        mbar_expect_tx(&bars[0], 4 * kBox);
        tma_load_3d(sm + L::kC, &tm_c, g * kN, k * kBlk, b, &bars[0]);
        tma_load_3d(sm + L::kC + kBox, &tm_c, g * kN + 64, k * kBlk, b, &bars[0]);
        tma_load_3d(sm + L::kB, &tm_b, g * kN, k * kBlk, b, &bars[0]);
        tma_load_3d(sm + L::kB + kBox, &tm_b, g * kN + 64, k * kBlk, b, &bars[0]);
        ok = mbar_wait(&bars[0], 0, err);
        if (ok) {
            tc_fence_after();
            const uint32_t aC = smem_u32(sm + L::kC), aB = smem_u32(sm + L::kB);
            constexpr uint32_t idG = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kb = ks >> 2, off = (ks & 3) * 32;
                umma_f16(tmem, smem_desc_sw128(aC + kb * kBox + off, 16, 1024),
                         smem_desc_sw128(aB + kb * kBox + off, 16, 1024), idG, ks > 0 ? 1u : 0u);
            }
            umma_commit(&bars[1]);
        }
    }
    ok = named_bar_and(1, kGramThreads, ok);
    if (ok) ok = mbar_wait(&bars[1], 0, err);
    tc_fence_after();
    const int r = warp * 32 + lane;
    uint4* out = gram + ((size_t)(b * ngroups + g) * nblocks + k) * (kGramBytes / 16);
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + kc * 32, v);
        tmem_wait_ld();
        if (ok) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int e = 8 * c;
                out[(kc * kBlk + r) * 4 + c] = make_uint4(
                    pack_bf16x2(__uint_as_float(v[e + 0]), __uint_as_float(v[e + 1])),
                    pack_bf16x2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                    pack_bf16x2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                    pack_bf16x2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
            }
        }
    }
    // the decay factors come from the kernel before this one; when this grid completes, that
    // one has completed too, so the chain kernel after it may read both
    griddep_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ================================================================ chain kernel
constexpr int kChainThreads = 640;
constexpr int kMaxHeads = 3;                    // heads per CTA (their states share TMEM)
constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpConv = 2, kWarpP0 = 4, kWarpE0 = 12, kWarpG0 = 16;
constexpr int kConvThreads = 64, kPThreads = 256;

// TMEM columns: the heads' states, the two P buffers (bf16 pairs), Yo, Yd, C_k (bf16 pairs)
constexpr uint32_t kColH = 0, kColP = 192, kColYo = 320, kColYd = 448;   // Yo: two buffers

struct ChainSmem {
    static constexpr int kXSlots = 4;
    static constexpr int kCst = 0;                       // C_k staging [2 n-halves][128 rows][128 B]
    static constexpr int kB0 = kCst + 2 * kBox;          // B_k ring: 2 x [2 n-halves][128 rows][128 B]
    static constexpr int kXt0 = kB0 + 4 * kBox;          // X~ ring: 2 x [128 rows][128 B]
    static constexpr int kImg = kXt0 + 2 * kBox;         // bf16 state image (MN-major, 64-byte swizzle)
    static constexpr int kSlot0 = kImg + kHImage;        // item slots:
    static constexpr int kXo = 0;                        //   x (then y) [128 rows][128 B]
    static constexpr int kLo = kBox;                     //   Lam[128]
    static constexpr int kDo = kLo + 512;                //   dt[128]
    static constexpr int kVo = kDo + 512;                //   column factors, sub-block-end reference
    static constexpr int kWo = kVo + 512;                //   column factors, sub-block-start reference
    static constexpr int kSlotBytes = kBox + 2048;
    static constexpr int kBar = kSlot0 + kXSlots * kSlotBytes;
    static constexpr int kNumBars = 32;
    static constexpr int kTslot = kBar + kNumBars * 8;
    static constexpr int kAbort = kTslot + 4;
    static constexpr int kBytes = kAbort + 12 + 1024;
};
static_assert(ChainSmem::kSlotBytes % 1024 == 0, "slots keep 1024-byte alignment");
static_assert(ChainSmem::kBytes <= 227 * 1024, "chain shared memory");

enum {
    CB_CSTAGED = 0, CB_CFREE,
    CB_BFULL, CB_BEMPTY = CB_BFULL + 2,
    CB_XFULL = CB_BEMPTY + 2, CB_XEMPTY = CB_XFULL + ChainSmem::kXSlots,
    CB_CONV = CB_XEMPTY + ChainSmem::kXSlots, CB_XTEMPTY = CB_CONV + 2,
    CB_UPD = CB_XTEMPTY + 2, CB_SDONE,
    CB_YOFULL = CB_SDONE + kMaxHeads, CB_YOEMPTY = CB_YOFULL + 2, CB_YDFULL = CB_YOEMPTY + 2, CB_YDPRIMED,
    CB_PFULL, CB_PEMPTY = CB_PFULL + 2, CB_COUNT = CB_PEMPTY + 2
};
static_assert(CB_COUNT <= ChainSmem::kNumBars, "chain barriers");

// x * w for the eight bf16 values of one 16-byte chunk, rounded to fp16
__device__ __forceinline__ uint4 scale_to_f16x8(uint4 u, float w) {
    u.x = pack_f16x2(bf16lo(u.x) * w, bf16hi(u.x) * w);
    u.y = pack_f16x2(bf16lo(u.y) * w, bf16hi(u.y) * w);
    u.z = pack_f16x2(bf16lo(u.z) * w, bf16hi(u.z) * w);
    u.w = pack_f16x2(bf16lo(u.w) * w, bf16hi(u.w) * w);
    return u;
}

// A diagonal sub-block with strong decay inside it: one exponential per element.  Rare, and
// kept out of line so that it does not take room in the instruction cache.
__device__ __noinline__ void p_subblock_strong_decay(uint32_t taddr, uint4 g0, uint4 g1, uint4 g2, uint4 g3,
                                                     int s0, int r, const float* sLam, const float* sDt)
{
    const uint32_t gw[16] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w,
                             g2.x, g2.y, g2.z, g2.w, g3.x, g3.y, g3.z, g3.w};
    const float lam_t = sLam[r];
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const int sa = s0 + 2 * e, sb = sa + 1;
        const float pa = sa <= r ? bf16lo(gw[e]) * expf(lam_t - sLam[sa]) * sDt[sa] : 0.f;
        const float pb = sb <= r ? bf16hi(gw[e]) * expf(lam_t - sLam[sb]) * sDt[sb] : 0.f;
        pk[e] = pack_bf16x2(pa, pb);
    }
    tmem_st16(taddr, pk);
}

// Bounded wait (as mbar_wait_or_abort), one out-of-line copy for all the kernel's call sites.
__device__ __noinline__ bool chain_wait(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag)
{
    return mbar_wait_or_abort(bar, parity, err, abort_flag);
}

// One 32-column sub-block of row r of P = G o exp(Lam_t - Lam_s) o dt_s (s <= t), from 16
// bf16 pairs of G, stored to TMEM at taddr (warp-collective; the sub-block is below, on or
// above the diagonal for the warp's 32 rows alike).  Below-diagonal sub-blocks use
// exp(Lam_t - Lam_q) exp(Lam_q - Lam_s), q the sub-block's last column; sub-blocks on the
// diagonal use the first column as reference when their own decay is below 40 (both factors
// within e^+-40) and one exponential per element otherwise.
__device__ __forceinline__ void p_store_subblock(uint32_t taddr, uint4 g0, uint4 g1, uint4 g2, uint4 g3, int s0,
                                              int r, const float* sLam, const float* sDt, const float* sV,
                                              const float* sW)
{
    const uint32_t gw[16] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w,
                             g2.x, g2.y, g2.z, g2.w, g3.x, g3.y, g3.z, g3.w};
    const float lam_t = sLam[r];
    uint32_t pk[16];
    // the branch is the same for the whole warp (rows r0 .. r0 + 31): tcgen05.st is warp-collective
    const int r0 = r & ~31;
    if (s0 + 32 <= r0) {
        const float u = expf(lam_t - sLam[s0 + 31]);
#pragma unroll
        for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(bf16lo(gw[e]) * u * sV[s0 + 2 * e], bf16hi(gw[e]) * u * sV[s0 + 2 * e + 1]);
    } else if (s0 >= r0 + 32) {
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = 0u;
    } else if (sLam[s0] - sLam[s0 + 31] < 40.f) {
        const float u = expf(lam_t - sLam[s0]);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int sa = s0 + 2 * e;
            const float pa = bf16lo(gw[e]) * u * sW[sa];
            const float pb = bf16hi(gw[e]) * u * sW[sa + 1];
            pk[e] = pack_bf16x2(sa <= r ? pa : 0.f, sa + 1 <= r ? pb : 0.f);
        }
    } else {
        p_subblock_strong_decay(taddr, g0, g1, g2, g3, s0, r, sLam, sDt);
        return;
    }
    tmem_st16(taddr, pk);
}

__global__ void __launch_bounds__(kChainThreads, 1)
chain_prefill_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b16,
                     const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                     const float* __restrict__ fac, const uint4* __restrict__ gram,
                     const float* __restrict__ D, const float* __restrict__ init_state,
                     float* __restrict__ final_state, int seqlen, int nheads, int ngroups, int nblk,
                     int ctas_per_group, int* err)
{
    using L = ChainSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kTslot);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kAbort);

    // this CTA's heads: hlo .. hlo + nh - 1 of group g of batch b
    const int hpg = nheads / ngroups;
    const int unit = blockIdx.x / ctas_per_group, part = blockIdx.x - unit * ctas_per_group;
    const int b = unit / ngroups, g = unit - b * ngroups;
    const int hlo = g * hpg + (part * hpg) / ctas_per_group;
    const int nh = g * hpg + ((part + 1) * hpg) / ctas_per_group - hlo;     // 1 .. kMaxHeads
    const int total = nblk * nh;                       // items (k, j), i = k nh + j
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        mbar_init(&bars[CB_CSTAGED], 1);
        mbar_init(&bars[CB_CFREE], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[CB_BFULL + i], 1);
            mbar_init(&bars[CB_BEMPTY + i], 1);
            mbar_init(&bars[CB_CONV + i], 2);
            mbar_init(&bars[CB_XTEMPTY + i], 1);
            mbar_init(&bars[CB_PFULL + i], kPThreads);
            mbar_init(&bars[CB_PEMPTY + i], 1);
        }
        for (int i = 0; i < L::kXSlots; ++i) {
            mbar_init(&bars[CB_XFULL + i], 1);
            mbar_init(&bars[CB_XEMPTY + i], 4);
        }
        mbar_init(&bars[CB_UPD], 4);
        for (int i = 0; i < kMaxHeads; ++i) mbar_init(&bars[CB_SDONE + i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[CB_YOFULL + i], 1);
            mbar_init(&bars[CB_YOEMPTY + i], 4);
        }
        mbar_init(&bars[CB_YDFULL], 1);
        mbar_init(&bars[CB_YDPRIMED], 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    auto slot = [&](int i) { return sm + L::kSlot0 + (i & (L::kXSlots - 1)) * L::kSlotBytes; };
    // bounded wait, the same answer for the whole warp (tcgen05.ld / st are warp-collective)
    auto wait_warp = [&](int bar, uint32_t parity) {
        const bool ok = chain_wait(&bars[bar], parity, err, abort_flag);
        return __all_sync(0xffffffffu, ok);
    };

    if (warp == kWarpLoad) {
        if (lane == 0) {
            // ------------------------------------------------ x and decay factors, one slot per item
            griddep_wait();                              // the decay factors come from an earlier kernel
            int issued = 0;
            for (int i = 0; i < total; ++i) {
                const int k = i / nh, h = hlo + (i - k * nh);
                if (i >= L::kXSlots &&
                    !mbar_wait_or_abort(&bars[CB_XEMPTY + (i & 3)], ((i >> 2) - 1) & 1, err, abort_flag))
                    break;
                uint8_t* sl = slot(i);
                mbar_expect_tx(&bars[CB_XFULL + (i & 3)], kBox + 4 * 512);
                tma_load_3d(sl + L::kXo, &tm_x, h * kP, k * kBlk, b, &bars[CB_XFULL + (i & 3)]);
                bulk_load(sl + L::kLo, fac + ((size_t)(b * nheads + h) * nblk + k) * 4 * kBlk, 4 * 512,
                          &bars[CB_XFULL + (i & 3)]);
                issued = i + 1;
            }
            // the CTA does not exit with loads in flight
            for (int i = max(0, issued - L::kXSlots); i < issued; ++i)
                mbar_wait(&bars[CB_XFULL + (i & 3)], (i >> 2) & 1, err);
        } else if (lane == 1) {
            // ------------------------------------------------ C_k (staging) and B_k (two-deep ring)
            griddep_wait();                              // the fp16 copy of B comes from an earlier kernel
            int kc = 0, kb = 0;
            for (int k = 0; k < nblk; ++k) {
                // every Yo of block k - 1 has read the staged C
                if (k >= 1 && !mbar_wait_or_abort(&bars[CB_CFREE], (k - 1) & 1, err, abort_flag)) break;
                mbar_expect_tx(&bars[CB_CSTAGED], 2 * kBox);
                tma_load_3d(sm + L::kCst, &tm_c, g * kN, k * kBlk, b, &bars[CB_CSTAGED]);
                tma_load_3d(sm + L::kCst + kBox, &tm_c, g * kN + 64, k * kBlk, b, &bars[CB_CSTAGED]);
                kc = k + 1;
                if (k >= 2 && !mbar_wait_or_abort(&bars[CB_BEMPTY + (k & 1)], ((k >> 1) - 1) & 1, err, abort_flag))
                    break;
                uint8_t* sb = sm + L::kB0 + (k & 1) * 2 * kBox;
                mbar_expect_tx(&bars[CB_BFULL + (k & 1)], 2 * kBox);
                tma_load_3d(sb, &tm_b16, g * kN, k * kBlk, b, &bars[CB_BFULL + (k & 1)]);
                tma_load_3d(sb + kBox, &tm_b16, g * kN + 64, k * kBlk, b, &bars[CB_BFULL + (k & 1)]);
                kb = k + 1;
            }
            if (kc > 0) mbar_wait(&bars[CB_CSTAGED], (kc - 1) & 1, err);
            for (int k = max(0, kb - 2); k < kb; ++k) mbar_wait(&bars[CB_BFULL + (k & 1)], (k >> 1) & 1, err);
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issue, two polled streams
            constexpr uint32_t idO = idesc_bf16_f32(128, 64, false, true);   // A in TMEM, B MN-major
            constexpr uint32_t idS = idesc_f16_f32(128, 64, true, true);     // A = B_k^T, B = X~: fp16, MN-major
            const uint32_t aImg = smem_u32(sm + L::kImg), aC = smem_u32(sm + L::kCst);
            int ia = 0, ib = 0;
            uint32_t idle = 0;
            while (ib < total) {
                bool progressed = false;
                if (ia < total) {
                    // Yo_i = C_k H^T and S_i = B_k^T X~_i (onto the head's state)
                    const int k = ia / nh, j = ia - k * nh;
                    if (mbar_test_wait(&bars[CB_UPD], ia & 1) &&
                        mbar_test_wait(&bars[CB_CONV + (ia & 1)], (ia >> 1) & 1) &&
                        (ia < 2 || mbar_test_wait(&bars[CB_YOEMPTY + (ia & 1)], ((ia >> 1) - 1) & 1)) &&
                        (j != 0 || (mbar_test_wait(&bars[CB_CSTAGED], k & 1) &&
                                    mbar_test_wait(&bars[CB_BFULL + (k & 1)], (k >> 1) & 1)))) {
                        tc_fence_after();
                        // Yo into buffer ia mod 2: A = C_k (shared memory, K-major over n)
#pragma unroll 1
                        for (int ks = 0; ks < 8; ++ks) {
                            const uint32_t kb = ks >> 2, off = (ks & 3) * 32;
                            umma_f16(tmem + kColYo + 64 * (ia & 1), smem_desc_sw128(aC + kb * kBox + off, 16, 1024),
                                     smem_desc_sw64(aImg + ks * 1024, 8192, 512), idO, ks > 0 ? 1u : 0u);
                        }
                        umma_commit(&bars[CB_YOFULL + (ia & 1)]);
                        if (j == nh - 1) umma_commit(&bars[CB_CFREE]);
                        const uint32_t aB = smem_u32(sm + L::kB0 + (k & 1) * 2 * kBox);
                        const uint32_t aXt = smem_u32(sm + L::kXt0 + (ia & 1) * kBox);
#pragma unroll 1
                        for (int ks = 0; ks < 8; ++ks)
                            umma_f16(tmem + kColH + 64 * j, smem_desc_sw128(aB + ks * 2048, kBox, 1024),
                                     smem_desc_sw128(aXt + ks * 2048, kBox, 1024), idS, 1u);
                        umma_commit(&bars[CB_SDONE + j]);
                        umma_commit(&bars[CB_XTEMPTY + (ia & 1)]);
                        if (j == nh - 1) umma_commit(&bars[CB_BEMPTY + (k & 1)]);
                        ++ia;
                        progressed = true;
                    }
                }
                if (ib < ia) {
                    // y_i = (exp(Lam_t) Yo_i + D x_i) + P_i X_i, onto the epilogue's first half
                    if (mbar_test_wait(&bars[CB_PFULL + (ib & 1)], (ib >> 1) & 1) &&
                        mbar_test_wait(&bars[CB_YDPRIMED], ib & 1)) {
                        tc_fence_after();
                        const uint32_t aX = smem_u32(slot(ib) + L::kXo);
#pragma unroll 1
                        for (int ks = 0; ks < 8; ++ks)
                            umma_f16_ts(tmem + kColYd, tmem + kColP + 64 * (ib & 1) + ks * 8,
                                        smem_desc_sw128(aX + ks * 2048, kBox, 1024), idO, 1u);
                        umma_commit(&bars[CB_PEMPTY + (ib & 1)]);
                        umma_commit(&bars[CB_YDFULL]);
                        ++ib;
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = 0;
                } else if (++idle >= (1u << 24) || ((idle & 1023u) == 0 && *abort_flag)) {
                    if (idle >= (1u << 24)) {
                        record_error(err, SSD_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    break;
                }
            }
            // the CTA does not release TMEM with MMAs in flight
            if (ib > 0) mbar_wait(&bars[CB_YDFULL], (ib - 1) & 1, err);
            if (ia > ib) mbar_wait(&bars[CB_XTEMPTY + ((ia - 1) & 1)], ((ia - 1) >> 1) & 1, err);
        }
    } else if (warp < kWarpP0) {
        // ---------------------------------------------------- X~ = w o X (fp16), w_s = exp(Lam_end - Lam_s) dt_s
        const int cid = tid - kWarpConv * 32;
        for (int i = 0; i < total; ++i) {
            if (!wait_warp(CB_XFULL + (i & 3), (i >> 2) & 1)) break;
            if (i >= 2 && !wait_warp(CB_XTEMPTY + (i & 1), ((i >> 1) - 1) & 1)) break;
            const uint8_t* sl = slot(i);
            const float* sLam = reinterpret_cast<const float*>(sl + L::kLo);
            const float* sDt = reinterpret_cast<const float*>(sl + L::kDo);
            const float lend = sLam[kBlk - 1];
            uint8_t* xt = sm + L::kXt0 + (i & 1) * kBox;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int row = cid + rr * kConvThreads;
                const float w = expf(lend - sLam[row]) * sDt[row];
                const uint4* src = reinterpret_cast<const uint4*>(sl + L::kXo + row * 128);
                uint4* dst = reinterpret_cast<uint4*>(xt + row * 128);
                uint4 u[8];
                // element-wise, so the chunks may be taken in any order: rotating by the row
                // keeps the eight threads of a shared-memory phase on distinct banks
#pragma unroll
                for (int c = 0; c < 8; ++c) u[c] = src[(c + row) & 7];
#pragma unroll
                for (int c = 0; c < 8; ++c) dst[(c + row) & 7] = scale_to_f16x8(u[c], w);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CB_CONV + (i & 1)]);
        }
    } else if (warp < kWarpE0) {
        // ---------------------------------------------------- P = G_k o exp(Lam_t - Lam_s) o dt_s, s <= t
        // Thread (row r, column half): G_k's 32-column sub-blocks kc0 = half and kc1 = half + 2
        // of row r, as bf16 pairs, read from global memory a block ahead into the other of
        // two register sets.
        const int pw = warp - kWarpP0;
        const int q = warp & 3, colhalf = pw >> 2;
        const int r = q * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        const int kc0 = colhalf, kc1 = colhalf + 2;
        const uint4* gbase = gram + (size_t)(b * ngroups + g) * nblk * (kGramBytes / 16);
        auto load_g = [&](int k, uint4 (&gv)[8]) {
            const uint4* gk = gbase + (size_t)k * (kGramBytes / 16);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                gv[c] = gk[(kc0 * kBlk + r) * 4 + c];
                gv[4 + c] = gk[(kc1 * kBlk + r) * 4 + c];
            }
        };
        griddep_wait();                                  // G comes from the kernel before this one
        uint4 ga[8], gb[8];
        if (nblk > 0) load_g(0, ga);
        if (nblk > 1) load_g(1, gb);
        bool live = true;
        for (int k = 0; k < nblk && live; ++k) {
            const bool odd = k & 1;
            for (int j = 0; j < nh; ++j) {
                const int i = k * nh + j, p = i & 1;
                live = wait_warp(CB_XFULL + (i & 3), (i >> 2) & 1) &&
                       (i < 2 || wait_warp(CB_PEMPTY + p, ((i >> 1) - 1) & 1));
                if (!live) break;
                const uint8_t* sl = slot(i);
                const float* sLam = reinterpret_cast<const float*>(sl + L::kLo);
                const float* sDt = reinterpret_cast<const float*>(sl + L::kDo);
                const float* sV = reinterpret_cast<const float*>(sl + L::kVo);
                const float* sW = reinterpret_cast<const float*>(sl + L::kWo);
                const uint32_t pc = trow + kColP + 64 * p;       // tokens 32 kc .. 32 kc + 31 at pc + 16 kc
                // one copy of the sub-block code (the kernel's roles run different code at once,
                // and its instruction footprint is what limits it)
#pragma unroll 1
                for (int w2 = 0; w2 < 2; ++w2) {
                    const int kc = w2 ? kc1 : kc0, o = 4 * w2;
                    p_store_subblock(pc + kc * 16, odd ? gb[o] : ga[o], odd ? gb[o + 1] : ga[o + 1],
                                     odd ? gb[o + 2] : ga[o + 2], odd ? gb[o + 3] : ga[o + 3], kc * 32, r,
                                     sLam, sDt, sV, sW);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[CB_PFULL + p]);
            }
            // block k + 2 into the register set block k used
            if (live && k + 2 < nblk) {
                if (odd) load_g(k + 2, gb);
                else load_g(k + 2, ga);
            }
        }
    } else if (warp < kWarpG0) {
        // ---------------------------------------------------- epilogue (thread r: token t = r)
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        // D of the CTA's heads, read once (a global load per item would sit on the item chain)
        float Dv[kMaxHeads];
#pragma unroll
        for (int j = 0; j < kMaxHeads; ++j) Dv[j] = j < nh ? D[hlo + j] : 0.f;

        for (int i = 0; i < total; ++i) {
            const int k = i / nh, j = i - k * nh;
            // exp(Lam_t) Yo + D x into the Yd accumulator, onto which the MMA then adds P X
            // (no partial result waits in registers); frees Yo
            if (!wait_warp(CB_YOFULL + (i & 1), (i >> 1) & 1)) break;
            tc_fence_after();
            uint8_t* sl = slot(i);
            const float u = expf(reinterpret_cast<const float*>(sl + L::kLo)[r]);
            const float Dh = j == 0 ? Dv[0] : (j == 1 ? Dv[1] : Dv[2]);
            uint8_t* xrow = sl + L::kXo + r * 128;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld32(tl + kColYo + 64 * (i & 1) + 32 * half, v);
                tmem_wait_ld();
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int qx = half * 4 + qq;
                    const uint4 xu = *reinterpret_cast<const uint4*>(xrow + ((qx ^ (r & 7)) << 4));
                    const uint32_t xw[4] = {xu.x, xu.y, xu.z, xu.w};
#pragma unroll
                    for (int k2 = 0; k2 < 4; ++k2) {
                        const int jj = qq * 8 + 2 * k2;
                        v[jj] = __float_as_uint(fmaf(u, __uint_as_float(v[jj]), Dh * bf16lo(xw[k2])));
                        v[jj + 1] = __float_as_uint(fmaf(u, __uint_as_float(v[jj + 1]), Dh * bf16hi(xw[k2])));
                    }
                }
                tmem_st16(tl + kColYd + 32 * half, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                tmem_st16(tl + kColYd + 32 * half + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[CB_YOEMPTY + (i & 1)]);
                mbar_arrive(&bars[CB_YDPRIMED]);
            }
            // y = the finished accumulator -> bf16, written over the item's x rows
            if (!wait_warp(CB_YDFULL, i & 1)) break;
            tc_fence_after();
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld32(tl + kColYd + 32 * half, v);
                tmem_wait_ld();
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int qx = half * 4 + qq;
                    uint32_t o[4];
#pragma unroll
                    for (int k2 = 0; k2 < 4; ++k2)
                        o[k2] = pack_bf16x2(__uint_as_float(v[qq * 8 + 2 * k2]), __uint_as_float(v[qq * 8 + 2 * k2 + 1]));
                    *reinterpret_cast<uint4*>(xrow + ((qx ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            tc_fence_before();
            // this warp's 32 rows of y (rows past seqlen are not written)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (k * kBlk + 32 * q < seqlen)
                    tma_store_3d(&tm_y, (hlo + j) * kP, k * kBlk + 32 * q, b, sl + L::kXo + q * 32 * 128);
                bulk_commit_group();
                bulk_wait_group_read1();                 // the previous item's rows have been read
                if (i > 0) mbar_arrive(&bars[CB_XEMPTY + ((i - 1) & 3)]);
            }
        }
        if (lane == 0) bulk_wait_group0();
    } else {
        // ---------------------------------------------------- states (thread n: state row n)
        const int q = warp & 3;
        const int n = q * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);

        // initial states: H_j[n][p] in TMEM lane n, column 64 j + p
        for (int j = 0; j < nh; ++j) {
            const float* is = init_state ? init_state + (size_t)(b * nheads + hlo + j) * kP * kN : nullptr;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = is ? __float_as_uint(is[(size_t)(16 * c + e) * kN + n]) : 0u;
                tmem_st16(tl + kColH + 64 * j + 16 * c, v);
            }
        }
        tmem_wait_st();
        tc_fence_before();

        bool live = true;
        for (int i = 0; i < total && live; ++i) {
            const int k = i / nh, j = i - k * nh;
            // the image buffer is free once Yo of item i - 1 is done
            if (i > 0 && !wait_warp(CB_YOFULL + ((i - 1) & 1), ((i - 1) >> 1) & 1)) { live = false; break; }
            // the bf16 image of H_k (operand of Yo), then H <- exp(Lam_end) H, onto which S
            // accumulates.  Image row n holds p in two 64-byte halves, 16-byte chunk jj of a
            // half stored at jj ^ ((n / 2) mod 4) (the 64-byte swizzle of the MN-major operand).
            if (!wait_warp(CB_XFULL + (i & 3), (i >> 2) & 1)) { live = false; break; }
            if (k > 0 && !wait_warp(CB_SDONE + j, (k - 1) & 1)) { live = false; break; }
            tc_fence_after();
            const float e = expf(reinterpret_cast<const float*>(slot(i) + L::kLo)[kBlk - 1]);
            const uint32_t hc = tl + kColH + 64 * j;
            uint8_t* img = sm + L::kImg + n * 64;
            const int sw = (n >> 1) & 3;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld32(hc + 32 * half, v);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint32_t* h8 = &v[8 * jj];
                    *reinterpret_cast<uint4*>(img + half * 8192 + ((jj ^ sw) << 4)) = make_uint4(
                        pack_bf16x2(__uint_as_float(h8[0]), __uint_as_float(h8[1])),
                        pack_bf16x2(__uint_as_float(h8[2]), __uint_as_float(h8[3])),
                        pack_bf16x2(__uint_as_float(h8[4]), __uint_as_float(h8[5])),
                        pack_bf16x2(__uint_as_float(h8[6]), __uint_as_float(h8[7])));
                }
#pragma unroll
                for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(e * __uint_as_float(v[c]));
                tmem_st16(hc + 32 * half, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                tmem_st16(hc + 32 * half + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            }
            tmem_wait_st();
            fence_proxy_async_smem();                    // image -> visible to the tensor cores
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CB_UPD]);
        }
        // final states, once each head's last S has accumulated
        for (int j = 0; j < nh && live; ++j) {
            if (!wait_warp(CB_SDONE + j, (nblk - 1) & 1)) break;
            tc_fence_after();
            float* fs = final_state + (size_t)(b * nheads + hlo + j) * kP * kN;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld32(tl + kColH + 64 * j + 32 * half, v);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) fs[(size_t)(32 * half + c) * kN + n] = __uint_as_float(v[c]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// CTAs per (b, g): at most three heads each, and as many as fill the SMs otherwise (never
// more than there are heads)
int chain_ctas_per_group(const Dims& d)
{
    const int hpg = d.nheads / d.ngroups;
    const int units = d.batch * d.ngroups;
    int cpg = (hpg + kMaxHeads - 1) / kMaxHeads;
    cpg = max(cpg, tc_sm_count() / max(units, 1));
    return min(cpg, hpg);
}

}  // namespace

cudaError_t launch_block_gram(const Dims& d, const void* B, const void* C, const TcWorkspace& w,
                              cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    if (d.chunk_len != kBlk || d.nseq != 0) return cudaErrorInvalidValue;
    CUtensorMap mb, mc;
    if (!tc_make_map(&mb, B, (uint64_t)d.ngroups * kN, d.seqlen, d.batch) ||
        !tc_make_map(&mc, C, (uint64_t)d.ngroups * kN, d.seqlen, d.batch))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(block_gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         GramSmem::kBytes);
    if (e != cudaSuccess) return e;
    return launch_dependent(block_gram_kernel, dim3(d.nchunks, d.ngroups, d.batch), dim3(kGramThreads),
                            GramSmem::kBytes, s, mb, mc, w.gram, d.ngroups, d.nchunks, device_error_word());
}

cudaError_t launch_chain_prefill(const Dims& d, const void* x, const void* C, const float* D,
                                 const TcWorkspace& w, const float* init_state, float* final_state,
                                 void* y, cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    if (d.chunk_len != kBlk || d.nseq != 0) return cudaErrorInvalidValue;
    CUtensorMap mx, mb, mc, my;
    if (!tc_make_map(&mx, x, (uint64_t)d.nheads * kP, d.seqlen, d.batch) ||
        !tc_make_map(&mb, w.b16, (uint64_t)d.ngroups * kN, d.seqlen, d.batch, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !tc_make_map(&mc, C, (uint64_t)d.ngroups * kN, d.seqlen, d.batch) ||
        !tc_make_map(&my, y, (uint64_t)d.nheads * kP, d.seqlen, d.batch, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chain_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         ChainSmem::kBytes);
    if (e != cudaSuccess) return e;
    const int cpg = chain_ctas_per_group(d);
    const unsigned grid = (unsigned)(d.batch * d.ngroups * cpg);
    return launch_dependent(chain_prefill_kernel, dim3(grid), dim3(kChainThreads), ChainSmem::kBytes, s, mx,
                            mb, mc, my, static_cast<const float*>(w.fac), static_cast<const uint4*>(w.gram), D,
                            init_state, final_state, d.seqlen, d.nheads, d.ngroups, d.nchunks, cpg,
                            device_error_word());
}

}  // namespace ssd
