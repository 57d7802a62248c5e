// Fused tensor-core prefill on sm_100a: x is read once, y written once, and no state goes
// through HBM except where one CTA hands a chain over to the next.
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
// pair_chain_kernel works on head pairs: a unit is (b, g, heads h0, h0 + 1), and a step is
// one 128-token block of one unit.  The two heads share C_k, B_k and G_k, and their state
// and output GEMMs are one MMA each with the heads side by side along N (N = 128):
//   S      = B_k^T [X~_0 | X~_1]   onto the pair's states in TMEM (lane n, column 64 j + p)
//   Yo     = C_k [H_0 | H_1]       (the states' bf16 image in shared memory)
//   Yd_j   = P_j X_j               (P_j in TMEM, one per head)
// The steps of all units, unit-major, are cut into one contiguous range per CTA, so every
// CTA does the same number of blocks however the units divide among the SMs.  A range
// starts and ends inside a unit at most once each; the CTA runs the piece at its end first
// (a unit's first blocks), then its whole units, then the piece at its start (a unit's last
// blocks), whose start state the previous CTA has by then handed over through a global
// slot.  With at least one unit of blocks per CTA that hand-off is ready before it is
// needed; it is a bounded wait either way.
//
// Roles (512 threads, four warps per scheduler, so 128 registers a thread):
//   warp 0      TMA, polling three streams: x and the decay factors of each step (two slots,
//               fetched into L2 four steps ahead); fp16 B_k in 64-token stages (three deep); C_k
//   warps 1, 14, 15  tcgen05.mma issue, one stream each: S, Yo, Yd_j
//   warps 2-5   X~ = w o X (fp16) for the state GEMM; the epilogue of the previous step,
//               y = Yd + exp(Lam_t) Yo + D x, written over that step's x and TMA-stored
//   warps 6-13  per step, first the state of one head for the warp's 32 TMEM lanes (the
//               bf16 image of H, the operand of Yo, then H <- exp(Lam_end) H, onto which S
//               accumulates; start and end states at piece boundaries), then two of the
//               four 32-column sub-blocks of P_j for its 32 rows, from G_k (read from
//               global memory a step ahead) and the factors
// Every wait is bounded; expiry records SSD_ERR_TIMEOUT in the device error word and the
// CTA drains without further waiting.
#include <algorithm>

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
// chain kernel's P threads read them.  CTA (0, 0, 0) also clears the chain kernel's
// hand-off flags.
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
                  uint4* __restrict__ gram, int ngroups, int nblocks, int* __restrict__ flags, int nflags,
                  int* err)
{
    using L = GramSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kSlot);
    griddep_launch_dependents();

    const int k = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (flags && k == 0 && g == 0 && b == 0)
        for (int i = tid; i < nflags; i += kGramThreads) flags[i] = 0;
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

// ================================================================ the steps of a CTA
// Steps i = u nb + k (unit u, block k) of all units, unit-major; CTA c owns [a, e) with
// a = c W / S, e = (c + 1) W / S.  It runs them as up to three intervals: the piece of unit
// e / nb at its end (that unit's first blocks), the whole units, and the piece of unit a / nb
// at its start (that unit's last blocks).  A range inside one unit is one interval.
struct StepSeq {
    long long lo[3], hi[3];
    long long a, e;
    int nb;
    __device__ void init(int c, int S, long long units, int nblk) {
        nb = nblk;
        const long long W = units * nblk;
        a = (long long)c * W / S;
        e = (long long)(c + 1) * W / S;
        const long long ua = a / nb, ue = e / nb;
        const long long ka = a - ua * nb;
        for (int r = 0; r < 3; ++r) lo[r] = hi[r] = 0;
        if (e <= (ua + 1) * nb) {
            lo[0] = a;
            hi[0] = e;
        } else {
            lo[0] = ue * nb;
            hi[0] = e;
            lo[1] = ka ? (ua + 1) * nb : a;
            hi[1] = ue * nb;
            lo[2] = ka ? a : 0;
            hi[2] = ka ? (ua + 1) * nb : 0;
        }
    }
};

// unit u -> batch, group and the pair's first head (units are (b, g, pair), b-major)
struct UnitMap {
    int ngroups, hpg;
    __device__ void map(int u, int* b, int* g, int* h0) const {
        const int pairs = hpg >> 1;
        const int bg = u / pairs, pr = u - bg * pairs;
        *b = bg / ngroups;
        *g = bg - *b * ngroups;
        *h0 = *g * hpg + 2 * pr;
    }
};

// Walks a CTA's steps in order.  The current interval's bounds and the unit, block, batch,
// group and first head of the current step are kept in registers and advanced
// incrementally: the divisions that locate a step run only where an interval starts or the
// unit changes, not on every step.
struct StepIter {
    const StepSeq* q;
    UnitMap um;
    int r, nb;
    long long i, lo, hi;
    int u, k, b, g, h0;
    __device__ void start(const StepSeq& s, const UnitMap& m) {
        q = &s;
        um = m;
        nb = s.nb;
        r = -1;
        hi = 0;
        i = 0;
        advance();
    }
    // moves to the next non-empty interval (or past the last)
    __device__ void advance() {
        for (;;) {
            ++r;
            if (r >= 3) return;
            lo = r == 0 ? q->lo[0] : (r == 1 ? q->lo[1] : q->lo[2]);
            hi = r == 0 ? q->hi[0] : (r == 1 ? q->hi[1] : q->hi[2]);
            if (lo < hi) break;
        }
        i = lo;
        u = (int)(i / nb);
        k = (int)(i - (long long)u * nb);
        um.map(u, &b, &g, &h0);
    }
    __device__ bool valid() const { return r < 3; }
    __device__ void next() {
        ++i;
        if (i >= hi) {
            advance();
            return;
        }
        if (++k == nb) {
            k = 0;
            ++u;
            um.map(u, &b, &g, &h0);
        }
    }
    __device__ int unit() const { return u; }
    __device__ int block() const { return k; }
    __device__ bool first() const { return i == lo || k == 0; }
    __device__ bool last() const { return i == hi - 1 || k == nb - 1; }
};

// ================================================================ chain kernel
constexpr int kPairThreads = 512;
constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpE0 = 2, kWarpP0 = 6, kWarpMmaO = 14, kWarpMmaD = 15;
constexpr int kWarpMmaS = kWarpMma;
constexpr int kPThreads = 256;
constexpr int kHandoffArrivals = 8;             // one per P/state warp
constexpr int kPrefetchSteps = 4;               // steps of x fetched into L2 ahead of their loads

// TMEM columns: the pair's states (lane n), Yd of each head, Yo of the pair (lane t), the
// two P buffers (bf16 pairs, lane t)
constexpr uint32_t kColH = 0, kColYd = 128, kColYo = 256, kColP = 384;

struct PairSmem {
    static constexpr int kC = 0;                          // C_k [2 n-halves][128 t][128 B] bf16
    static constexpr int kBStages = 3;
    static constexpr int kBStage = 2 * 8192;              // fp16 B: [2 n-halves][64 t][128 B]
    static constexpr int kB0 = kC + 2 * kBox;
    static constexpr int kXSlots = 2;
    static constexpr int kFacBytes = 4 * 512;             // per head: Lam, dt, and two column-factor rows
    static constexpr int kXFac = 2 * kBox;                // in a slot: x of head 0, of head 1, then factors
    static constexpr int kXSlot = 2 * kBox + 2 * kFacBytes;
    static constexpr int kX0 = kB0 + kBStages * kBStage;
    static constexpr int kXt = kX0 + kXSlots * kXSlot;    // X~ [2 heads][128 t][128 B] fp16
    static constexpr int kImg = kXt + 2 * kBox;           // state images [2 heads][2 p-halves][128 n][64 B]
    static constexpr int kBar = kImg + 2 * kHImage;
    static constexpr int kNumBars = 24;
    static constexpr int kTslot = kBar + kNumBars * 8;
    static constexpr int kAbort = kTslot + 4;
    static constexpr int kBytes = kAbort + 12 + 1024;
};
static_assert(PairSmem::kXSlot % 1024 == 0 && PairSmem::kBStage % 1024 == 0, "1024-byte alignment");
static_assert(PairSmem::kBytes <= 227 * 1024, "chain shared memory");

enum {
    PB_XF = 0, PB_XE = PB_XF + PairSmem::kXSlots,
    PB_BF = PB_XE + PairSmem::kXSlots, PB_BE = PB_BF + PairSmem::kBStages,
    PB_CF = PB_BE + PairSmem::kBStages, PB_CE,
    PB_UPD, PB_CONV, PB_SD, PB_YO,
    PB_PF, PB_YD = PB_PF + 2, PB_EPI = PB_YD + 2, PB_COUNT = PB_EPI + 2
};
static_assert(PB_COUNT <= PairSmem::kNumBars, "chain barriers");

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
// Between polls the thread sleeps (64 ns, doubling to 512 ns): a dozen roles wait at any
// moment, and a spinning waiter takes issue slots from the warps that do the work.  Gives
// up after about 2^22 polls (seconds), or soon after another thread has recorded a timeout.
__device__ __noinline__ bool chain_wait(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag)
{
    if (mbar_try_wait(bar, parity)) return true;
    uint32_t ns = 64;
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        __nanosleep(ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (ns < 512) ns <<= 1;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    record_error(err, SSD_ERR_TIMEOUT);
    *abort_flag = 1;
    return false;
}

// Bounded spin until *flag >= value (acquire), giving up early once the CTA has aborted.
__device__ __noinline__ bool wait_handoff(const int* flag, int value, int* err, volatile int* abort_flag)
{
    for (uint32_t it = 0; it < (1u << 24); ++it) {
        if (ld_acquire_gpu(flag) >= value) return true;
        if ((it & 255u) == 255u && *abort_flag) return false;
        __nanosleep(64);
    }
    record_error(err, SSD_ERR_TIMEOUT);
    *abort_flag = 1;
    return false;
}

// Two bf16 products at once: (a.lo * b.lo, a.hi * b.hi), each rounded to bf16.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// One 32-column sub-block of row r of P = G o exp(Lam_t - Lam_s) o dt_s (s <= t), from 16
// bf16 pairs of G, stored to TMEM at taddr (warp-collective; the sub-block is below, on or
// above the diagonal for the warp's 32 rows alike).  The decay-times-dt factor of each
// element is formed in fp32, rounded to bf16 and multiplied into G two columns at a time
// (a second bf16 rounding of P, well inside the tolerance: the parity tests bound it).  Below-diagonal sub-blocks use
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
    const int r0 = r & ~31;
    if (s0 + 32 <= r0) {
        const float u = expf(lam_t - sLam[s0 + 31]);
        const float4* v4 = reinterpret_cast<const float4*>(sV + s0);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
            const float4 f = v4[e4];
            pk[2 * e4] = mul_bf16x2(gw[2 * e4], pack_bf16x2(u * f.x, u * f.y));
            pk[2 * e4 + 1] = mul_bf16x2(gw[2 * e4 + 1], pack_bf16x2(u * f.z, u * f.w));
        }
    } else if (s0 >= r0 + 32) {
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = 0u;
    } else if (sLam[s0] - sLam[s0 + 31] < 40.f) {
        const float u = expf(lam_t - sLam[s0]);
        const float4* w4 = reinterpret_cast<const float4*>(sW + s0);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
            const float4 f = w4[e4];
            const int sa = s0 + 4 * e4;
            pk[2 * e4] = mul_bf16x2(gw[2 * e4], pack_bf16x2(sa <= r ? u * f.x : 0.f, sa + 1 <= r ? u * f.y : 0.f));
            pk[2 * e4 + 1] = mul_bf16x2(gw[2 * e4 + 1],
                                        pack_bf16x2(sa + 2 <= r ? u * f.z : 0.f, sa + 3 <= r ? u * f.w : 0.f));
        }
    } else {
        p_subblock_strong_decay(taddr, g0, g1, g2, g3, s0, r, sLam, sDt);
        return;
    }
    tmem_st16(taddr, pk);
}

__global__ void __launch_bounds__(kPairThreads, 1)
pair_chain_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b16,
                  const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                  const float* __restrict__ fac,
                  const uint4* __restrict__ gram, const float* __restrict__ D,
                  const float* __restrict__ init_state, float* __restrict__ final_state,
                  __nv_bfloat16* __restrict__ y, float* __restrict__ handoff, int* __restrict__ handoff_flag,
                  int seqlen, int nheads, int ngroups, int nblk, int units, int* err)
{
    using L = PairSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kTslot);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kAbort);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cta = blockIdx.x, nctas = gridDim.x;

    StepSeq seq;
    seq.init(cta, nctas, units, nblk);
    const UnitMap um{ngroups, nheads / ngroups};
    const int total = (int)(seq.e - seq.a);               // steps of this CTA

    if (tid == 0) {
        for (int i = 0; i < L::kXSlots; ++i) {
            mbar_init(&bars[PB_XF + i], 1);
            mbar_init(&bars[PB_XE + i], 1 + 4);           // the last Yd MMA, the 4 epilogue warps
        }
        for (int i = 0; i < L::kBStages; ++i) {
            mbar_init(&bars[PB_BF + i], 1);
            mbar_init(&bars[PB_BE + i], 1);
        }
        mbar_init(&bars[PB_CF], 1);
        mbar_init(&bars[PB_CE], 1);
        mbar_init(&bars[PB_UPD], 8);
        mbar_init(&bars[PB_CONV], 4);
        mbar_init(&bars[PB_SD], 1);
        mbar_init(&bars[PB_YO], 1);
        for (int j = 0; j < 2; ++j) {
            mbar_init(&bars[PB_PF + j], kPThreads);
            mbar_init(&bars[PB_YD + j], 1);
            mbar_init(&bars[PB_EPI + j], 4);
        }
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

    auto xslot = [&](int s) { return sm + L::kX0 + (s & 1) * L::kXSlot; };
    auto facp = [&](int s, int j) { return reinterpret_cast<const float*>(xslot(s) + L::kXFac + j * L::kFacBytes); };
    auto wait_warp = [&](int bar, uint32_t parity) {
        const bool ok = chain_wait(&bars[bar], parity, err, abort_flag);
        return __all_sync(0xffffffffu, ok);
    };

    if (warp == kWarpLoad) {
        if (lane == 0) {
            // ------------------------------------------------ loads, three polled streams
            griddep_wait();                              // factors and fp16 B come from earlier kernels
            StepIter ix, ib, ic, ip;
            ix.start(seq, um);
            ib.start(seq, um);
            ic.start(seq, um);
            // x and the decay factors of the steps ahead are fetched into L2 first, so that a
            // slot's own load (issued once the slot is free) finds them there
            ip.start(seq, um);
            auto prefetch = [&](const StepIter& at) {
                const int b = at.b, g = at.g, h0 = at.h0;
                const int k = at.block();
                for (int j = 0; j < 2; ++j) {
                    tma_prefetch_3d(&tm_x, (h0 + j) * kP, k * kBlk, b);
                    bulk_prefetch_l2(fac + ((size_t)(b * nheads + h0 + j) * nblk + k) * 4 * kBlk, L::kFacBytes);
                }
            };
            for (int i = 0; i < kPrefetchSteps && ip.valid(); ++i, ip.next()) prefetch(ip);
            int nx = 0, nbh = 0, nc = 0;           // steps of x, 64-token halves of B, steps of C
            uint32_t idle = 0;
            while (ix.valid() || ib.valid() || ic.valid()) {
                bool progressed = false;
                if (ix.valid() && (nx < L::kXSlots ||
                                   mbar_test_wait(&bars[PB_XE + (nx & 1)], ((nx >> 1) - 1) & 1))) {
                    const int b = ix.b, g = ix.g, h0 = ix.h0;
                    const int k = ix.block();
                    uint8_t* sl = xslot(nx);
                    uint64_t* fb = &bars[PB_XF + (nx & 1)];
                    mbar_expect_tx(fb, 2 * kBox + 2 * L::kFacBytes);
                    for (int j = 0; j < 2; ++j) {
                        tma_load_3d(sl + j * kBox, &tm_x, (h0 + j) * kP, k * kBlk, b, fb);
                        bulk_load(sl + L::kXFac + j * L::kFacBytes,
                                  fac + ((size_t)(b * nheads + h0 + j) * nblk + k) * 4 * kBlk, L::kFacBytes, fb);
                    }
                    ++nx;
                    ix.next();
                    if (ip.valid()) {
                        prefetch(ip);
                        ip.next();
                    }
                    progressed = true;
                }
                if (ib.valid()) {
                    const int st = (int)(nbh % L::kBStages);
                    if (nbh < L::kBStages || mbar_test_wait(&bars[PB_BE + st], ((nbh / L::kBStages) - 1) & 1)) {
                        const int b = ib.b, g = ib.g, h0 = ib.h0;
                        const int half = (int)(nbh & 1);
                        mbar_expect_tx(&bars[PB_BF + st], L::kBStage);
                        tma_load_4d(sm + L::kB0 + st * L::kBStage, &tm_b16, 0, ib.block() * kBlk + half * 64, 2 * g, b,
                                    &bars[PB_BF + st]);
                        ++nbh;
                        if (half) ib.next();
                        progressed = true;
                    }
                }
                if (ic.valid() && (nc == 0 || mbar_test_wait(&bars[PB_CE], (nc - 1) & 1))) {
                    const int b = ic.b, g = ic.g, h0 = ic.h0;
                    mbar_expect_tx(&bars[PB_CF], 2 * kBox);
                    tma_load_3d(sm + L::kC, &tm_c, g * kN, ic.block() * kBlk, b, &bars[PB_CF]);
                    tma_load_3d(sm + L::kC + kBox, &tm_c, g * kN + 64, ic.block() * kBlk, b, &bars[PB_CF]);
                    ++nc;
                    ic.next();
                    progressed = true;
                }
                if (progressed) {
                    idle = 0;
                } else if (__nanosleep(128), ++idle >= (1u << 24) || ((idle & 1023u) == 0 && *abort_flag)) {
                    if (idle >= (1u << 24)) {
                        record_error(err, SSD_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    break;
                }
            }
            // the CTA does not exit with loads in flight
            for (int t = nx > L::kXSlots ? nx - L::kXSlots : 0; t < nx; ++t)
                mbar_wait(&bars[PB_XF + (t & 1)], (t >> 1) & 1, err);
            for (int h = nbh > L::kBStages ? nbh - L::kBStages : 0; h < nbh; ++h)
                mbar_wait(&bars[PB_BF + h % L::kBStages], (h / L::kBStages) & 1, err);
            if (nc > 0) mbar_wait(&bars[PB_CF], (nc - 1) & 1, err);
        }
    } else if (warp == kWarpMmaS) {
        if (lane == 0) {
            // ------------------------------------------------ S = B_k^T [X~_0 | X~_1] onto the states
            // A = fp16 B (MN-major, n-halves 8 KB apart), B = X~ (MN-major, heads 16 KB apart)
            constexpr uint32_t idS = idesc_f16_f32(128, 128, true, true);
            const uint32_t aXt = smem_u32(sm + L::kXt);
            int ns = 0;
            for (; ns < total; ++ns) {
                const int st0 = (int)((2 * ns) % L::kBStages), st1 = (int)((2 * ns + 1) % L::kBStages);
                if (!chain_wait(&bars[PB_UPD], ns & 1, err, abort_flag) ||
                    !chain_wait(&bars[PB_CONV], ns & 1, err, abort_flag) ||
                    !chain_wait(&bars[PB_BF + st0], ((2 * ns) / L::kBStages) & 1, err, abort_flag) ||
                    !chain_wait(&bars[PB_BF + st1], ((2 * ns + 1) / L::kBStages) & 1, err, abort_flag))
                    break;
                tc_fence_after();
#pragma unroll 1
                for (int ks = 0; ks < 8; ++ks) {
                    const int st = ks < 4 ? st0 : st1;
                    umma_f16(tmem + kColH,
                             smem_desc_sw128(smem_u32(sm + L::kB0 + st * L::kBStage) + (ks & 3) * 2048, 8192, 1024),
                             smem_desc_sw128(aXt + ks * 2048, kBox, 1024), idS, 1u);
                    if (ks == 3) umma_commit(&bars[PB_BE + st0]);
                }
                umma_commit(&bars[PB_BE + st1]);
                umma_commit(&bars[PB_SD]);
            }
            // the CTA does not release TMEM with MMAs in flight
            if (ns > 0) mbar_wait(&bars[PB_SD], (ns - 1) & 1, err);
        }
    } else if (warp == kWarpMmaO) {
        if (lane == 0) {
            // ------------------------------------------------ Yo = C_k [H_0 | H_1]
            // A = C (K-major), B = the images (MN-major, 64-byte swizzle, the four 32-column
            // blocks 8 KB apart); waits for the image (UPD), C, and the epilogue's reads of Yo
            constexpr uint32_t idO = idesc_bf16_f32(128, 128, false, true);
            const uint32_t aC = smem_u32(sm + L::kC), aImg = smem_u32(sm + L::kImg);
            int no = 0;
            for (; no < total; ++no) {
                if (!chain_wait(&bars[PB_UPD], no & 1, err, abort_flag) ||
                    !chain_wait(&bars[PB_CF], no & 1, err, abort_flag) ||
                    (no > 0 && (!chain_wait(&bars[PB_EPI], (no - 1) & 1, err, abort_flag) ||
                                !chain_wait(&bars[PB_EPI + 1], (no - 1) & 1, err, abort_flag))))
                    break;
                tc_fence_after();
#pragma unroll 1
                for (int ks = 0; ks < 8; ++ks)
                    umma_f16(tmem + kColYo, smem_desc_sw128(aC + (ks >> 2) * kBox + (ks & 3) * 32, 16, 1024),
                             smem_desc_sw64(aImg + ks * 1024, 8192, 512), idO, ks > 0 ? 1u : 0u);
                umma_commit(&bars[PB_CE]);
                umma_commit(&bars[PB_YO]);
            }
            if (no > 0) mbar_wait(&bars[PB_YO], (no - 1) & 1, err);
        }
    } else if (warp == kWarpMmaD) {
        if (lane == 0) {
            // ------------------------------------------------ Yd_j = P_j X_j
            constexpr uint32_t idD = idesc_bf16_f32(128, 64, false, true);
            int nd = 0;
            for (; nd < 2 * total; ++nd) {
                const int sd = nd >> 1;
                const int j = (int)(nd & 1);
                if (!chain_wait(&bars[PB_PF + j], sd & 1, err, abort_flag) ||
                    (sd > 0 && !chain_wait(&bars[PB_EPI + j], (sd - 1) & 1, err, abort_flag)) ||
                    !chain_wait(&bars[PB_XF + (sd & 1)], (sd >> 1) & 1, err, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t aX = smem_u32(xslot(sd) + j * kBox);
#pragma unroll 1
                for (int ks = 0; ks < 8; ++ks)
                    umma_f16_ts(tmem + kColYd + 64 * j, tmem + kColP + 64 * j + ks * 8,
                                smem_desc_sw128(aX + ks * 2048, kBox, 1024), idD, ks > 0 ? 1u : 0u);
                umma_commit(&bars[PB_YD + j]);
                if (j == 1) umma_commit(&bars[PB_XE + (sd & 1)]);
            }
            if (nd > 0) mbar_wait(&bars[PB_YD + ((nd - 1) & 1)], ((nd - 1) >> 1) & 1, err);
        }
    } else if (warp >= kWarpE0 && warp < kWarpP0) {
        // ---------------------------------------------------- X~, then the previous step's epilogue
        // Per step s: X~_s = w o X_s (the state GEMM's operand); then the epilogue of step
        // s - 1, y = Yd + exp(Lam_t) Yo + D x written over that step's x rows (each thread its
        // own row) and stored with one TMA store per warp and head; the slot is released once
        // the stores have read it.
        const int q = warp & 3;
        const int t = q * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        StepIter it;
        it.start(seq, um);
        int s = 0;
        int pb = 0, pk = 0, ph0 = 0;                     // the previous step: batch, block, first head
        float pD0 = 0.f, pD1 = 0.f;

        auto epilogue = [&](int ps) -> bool {
            if (!wait_warp(PB_YO, ps & 1)) return false;
            uint8_t* sl = xslot(ps);
            for (int j = 0; j < 2; ++j) {
                if (!wait_warp(PB_YD + j, ps & 1)) return false;
                tc_fence_after();
                const float u = expf(facp(ps, j)[t]);
                const float Dh = j ? pD1 : pD0;
                uint8_t* xrow = sl + j * kBox + t * 128;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    uint32_t yd[32], yo[32];
                    tmem_ld32(tl + kColYd + 64 * j + 32 * half, yd);
                    tmem_ld32(tl + kColYo + 64 * j + 32 * half, yo);
                    tmem_wait_ld();
                    if (half == 1) {
                        // Yd and Yo of head j have been read
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars[PB_EPI + j]);
                    }
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int cx = 4 * half + c4;                   // 16-byte chunk of the row
                        uint4* xp = reinterpret_cast<uint4*>(xrow + ((cx ^ (t & 7)) << 4));
                        const uint4 xu = *xp;
                        const uint32_t xw[4] = {xu.x, xu.y, xu.z, xu.w};
                        uint32_t o[4];
#pragma unroll
                        for (int k2 = 0; k2 < 4; ++k2) {
                            const int e = 8 * c4 + 2 * k2;
                            o[k2] = pack_bf16x2(
                                fmaf(u, __uint_as_float(yo[e]), __uint_as_float(yd[e])) + Dh * bf16lo(xw[k2]),
                                fmaf(u, __uint_as_float(yo[e + 1]), __uint_as_float(yd[e + 1])) + Dh * bf16hi(xw[k2]));
                        }
                        *xp = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                // this warp's 32 rows of y (rows past seqlen are not written)
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && pk * kBlk + 32 * q < seqlen)
                    tma_store_3d(&tm_y, (ph0 + j) * kP, pk * kBlk + 32 * q, pb, sl + j * kBox + q * 32 * 128);
            }
            if (lane == 0) {
                bulk_commit_group();
                bulk_wait_group_read0();                 // the stores have read the slot
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[PB_XE + (ps & 1)]);
            return true;
        };

        bool live = true;
        for (; it.valid() && live; it.next(), ++s) {
            const int b = it.b, h0 = it.h0;
            const int k = it.block();
            const float d0 = D[h0], d1 = D[h0 + 1];
            // X~_s: waits for the slot and for S of the previous step
            live = wait_warp(PB_XF + (s & 1), (s >> 1) & 1) && (s == 0 || wait_warp(PB_SD, (s - 1) & 1));
            if (!live) break;
            const uint8_t* sl = xslot(s);
#pragma unroll 1
            for (int j = 0; j < 2; ++j) {
                const float* sLam = facp(s, j);
                const float w = expf(sLam[kBlk - 1] - sLam[t]) * sLam[kBlk + t];
                const uint4* src = reinterpret_cast<const uint4*>(sl + j * kBox + t * 128);
                uint4* dst = reinterpret_cast<uint4*>(sm + L::kXt + j * kBox + t * 128);
                uint4 u8[8];
                // element-wise, so the chunks may be taken in any order: rotating by the row
                // keeps the eight threads of a shared-memory phase on distinct banks
#pragma unroll
                for (int c = 0; c < 8; ++c) u8[c] = src[(c + t) & 7];
#pragma unroll
                for (int c = 0; c < 8; ++c) dst[(c + t) & 7] = scale_to_f16x8(u8[c], w);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[PB_CONV]);
            if (s > 0) {
                live = epilogue(s - 1);
                if (!live) break;
            }
            pb = b;
            pk = k;
            ph0 = h0;
            pD0 = d0;
            pD1 = d1;
        }
        if (live && s > 0) epilogue(s - 1);
        if (lane == 0) bulk_wait_group0();
    } else if (warp >= kWarpP0 && warp < kWarpP0 + 8) {
        // ---------------------------------------------------- state of head c, then P_j
        // Warp (quarter q, c): TMEM lanes 32 q .. 32 q + 31.  The state part treats the lane as
        // state row n and owns head c's 64 columns; the P part treats it as row r of P_j and
        // builds G_k's 32-column sub-blocks kc0 = c and kc1 = c + 2, from bf16 pairs of G read
        // from global memory a step ahead.
        const int pw = warp - kWarpP0;
        const int q = warp & 3, c = pw >> 2;
        const int r = q * 32 + lane;                     // = n for the state part
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        const int kc0 = c, kc1 = c + 2;
        auto load_g = [&](const StepIter& at, uint4 (&gv)[8]) {
            const int b = at.b, g = at.g, h0 = at.h0;
            const uint4* gk = gram + ((size_t)(b * ngroups + g) * nblk + at.block()) * (kGramBytes / 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                gv[i] = gk[(kc0 * kBlk + r) * 4 + i];
                gv[4 + i] = gk[(kc1 * kBlk + r) * 4 + i];
            }
        };
        griddep_wait();                                  // G and the hand-off flags come from earlier kernels
        StepIter it;
        it.start(seq, um);
        // G of the current step; the next step's G is loaded once this step's P is built, and
        // lands while the next step's state update runs
        uint4 gv[8];
        if (it.valid()) load_g(it, gv);
        const uint32_t hc = tl + kColH + 64 * c;         // this warp's head's state columns
        const int sw = (r >> 1) & 3;
        int s = 0;
        bool live = true;
        for (; it.valid() && live; it.next(), ++s) {
            const int b = it.b, g = it.g, h0 = it.h0;
            const int k = it.block();
            // ---- state
            if (it.first()) {
                // start state: the initial state (or zeros) at block 0, else the previous CTA's hand-off
                const float* src = nullptr;
                if (k == 0) {
                    if (init_state) src = init_state + (size_t)(b * nheads + h0 + c) * kP * kN;
                } else {
                    live = __all_sync(0xffffffffu, lane != 0 ||
                                                   wait_handoff(&handoff_flag[cta], kHandoffArrivals, err, abort_flag));
                    if (!live) break;
                    (void)ld_acquire_gpu(&handoff_flag[cta]);     // every lane reads after an acquire
                    src = handoff + ((size_t)cta * 2 + c) * kP * kN;
                }
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t v[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        v[e] = src ? __float_as_uint(__ldcg(src + (size_t)(16 * cc + e) * kN + r)) : 0u;
                    tmem_st16(hc + 16 * cc, v);
                }
                tmem_wait_st();
            } else {
                live = wait_warp(PB_SD, (s - 1) & 1);
                if (!live) break;
            }
            // the image buffer is free once Yo of the previous step is done; the factors of this step
            live = (s == 0 || wait_warp(PB_YO, (s - 1) & 1)) && wait_warp(PB_XF + (s & 1), (s >> 1) & 1);
            if (!live) break;
            tc_fence_after();
            {
                // the bf16 image of H_k (operand of Yo), then H <- exp(Lam_end) H, onto which S
                // accumulates.  Image row n holds p in two 64-byte halves, 16-byte chunk jj of a
                // half stored at jj ^ ((n / 2) mod 4) (the 64-byte swizzle of the MN-major operand).
                const float e = expf(facp(s, c)[kBlk - 1]);
                uint8_t* img = sm + L::kImg + c * kHImage + r * 64;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {    // columns 32 half .. 32 half + 31
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
                    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(e * __uint_as_float(v[i]));
                    tmem_st16(hc + 32 * half, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                    tmem_st16(hc + 32 * half + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
                }
                tmem_wait_st();
                fence_proxy_async_smem();                // image -> visible to the tensor cores
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[PB_UPD]);
            }
            if (it.last()) {
                // end state, once S of this step has accumulated: the final state at the unit's
                // last block, else a hand-off to the next CTA.  The next piece's first step then
                // loads its start state over H without waiting for S again.
                live = wait_warp(PB_SD, s & 1);
                if (!live) break;
                tc_fence_after();
                const bool final_block = k == nblk - 1;
                float* dst = final_block ? final_state + (size_t)(b * nheads + h0 + c) * kP * kN
                                         : handoff + ((size_t)(cta + 1) * 2 + c) * kP * kN;
#pragma unroll 1
                for (int q16 = 0; q16 < 4; ++q16) {
                    uint32_t v[16];
                    tmem_ld16(hc + 16 * q16, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) dst[(size_t)(16 * q16 + e) * kN + r] = __uint_as_float(v[e]);
                }
                if (!final_block) {
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) atomicAdd(&handoff_flag[cta + 1], 1);
                }
                tc_fence_before();
            }
            // ---- P_j = G_k o exp(Lam_t - Lam_s) o dt_s, s <= t
            for (int j = 0; j < 2; ++j) {
                live = s == 0 || wait_warp(PB_YD + j, (s - 1) & 1);
                if (!live) break;
                const float* sLam = facp(s, j);
                const float* sDt = sLam + kBlk;
                const float* sV = sLam + 2 * kBlk;
                const float* sW = sLam + 3 * kBlk;
                const uint32_t pc = tl + kColP + 64 * j;         // tokens 32 kc .. 32 kc + 31 at pc + 16 kc
#pragma unroll 1
                for (int w2 = 0; w2 < 2; ++w2) {
                    const int kc = w2 ? kc1 : kc0;
                    // constant register indices (a computed index would put the set in local memory)
                    const uint4 g0 = w2 ? gv[4] : gv[0], g1 = w2 ? gv[5] : gv[1];
                    const uint4 g2 = w2 ? gv[6] : gv[2], g3 = w2 ? gv[7] : gv[3];
                    p_store_subblock(pc + kc * 16, g0, g1, g2, g3, kc * 32, r, sLam, sDt, sV, sW);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[PB_PF + j]);
            }
            // the next step's G
            if (live) {
                StepIter nx = it;
                nx.next();
                if (nx.valid()) load_g(nx, gv);
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

int pair_ctas(const Dims& d)
{
    const long long units = fused_units(d);
    return (int)std::min<long long>(std::min<long long>(units, tc_sm_count()), kFusedMaxCtas);
}

}  // namespace

bool fused_prefill_supported(const Dims& d)
{
    return d.nseq == 0 && (d.nheads / d.ngroups) % 2 == 0;
}

long long fused_units(const Dims& d)
{
    return (long long)d.batch * d.ngroups * ((d.nheads / d.ngroups) / 2);
}

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
    const int nflags = fused_prefill_supported(d) ? pair_ctas(d) + 1 : 0;
    return launch_dependent(block_gram_kernel, dim3(d.nchunks, d.ngroups, d.batch), dim3(kGramThreads),
                            GramSmem::kBytes, s, mb, mc, w.gram, d.ngroups, d.nchunks,
                            nflags ? w.handoff_flag : nullptr, nflags, device_error_word());
}

cudaError_t launch_chain_prefill(const Dims& d, const void* x, const void* C, const float* D,
                                 const TcWorkspace& w, const float* init_state, float* final_state,
                                 void* y, cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    if (d.chunk_len != kBlk || !fused_prefill_supported(d)) return cudaErrorInvalidValue;
    CUtensorMap mx, mb, mc, my;
    // fp16 B [b][T][G][N] seen as (n mod 64, t, 2 g + n / 64, b): a box is both n-halves of 64 rows
    const uint64_t T = d.seqlen, G = d.ngroups, Bt = d.batch;
    const uint64_t bdim[4] = {64, T, 2 * G, Bt};
    const uint64_t bstr[3] = {G * kN * 2, 128, T * G * kN * 2};
    const uint32_t bbox[4] = {64, 64, 2, 1};
    if (!tc_make_map(&mx, x, (uint64_t)d.nheads * kP, d.seqlen, d.batch) ||
        !tc_encode_map(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, w.b16, bdim, bstr, bbox, true) ||
        !tc_make_map(&mc, C, (uint64_t)d.ngroups * kN, d.seqlen, d.batch) ||
        !tc_make_map(&my, y, (uint64_t)d.nheads * kP, d.seqlen, d.batch, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(pair_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         PairSmem::kBytes);
    if (e != cudaSuccess) return e;
    const int ctas = pair_ctas(d);
    return launch_dependent(pair_chain_kernel, dim3(ctas), dim3(kPairThreads), PairSmem::kBytes, s, mx, mb, mc, my,
                            static_cast<const float*>(w.fac), static_cast<const uint4*>(w.gram), D, init_state,
                            final_state, static_cast<__nv_bfloat16*>(y), w.handoff, w.handoff_flag, d.seqlen,
                            d.nheads, d.ngroups, d.nchunks, (int)fused_units(d), device_error_word());
}

}  // namespace ssd
