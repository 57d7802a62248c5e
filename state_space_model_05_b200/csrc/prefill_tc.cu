// Tensor-core stages of the bf16 chunked SSD prefill on sm_100a: tcgen05.mma with
// TMEM accumulators, operands staged in shared memory by TMA.
//
// "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching for
// Inference", section "2. Metodologia": the SSD layer is dominated by matrix
// contractions inside fixed-size chunks, masked by a static lower-triangular decay
// mask whose exponents are taken in fp32, and chunks communicate only through an
// N x P state per (batch, head).  These stages work in 128-token blocks: a 256-token
// chunk is two blocks, and the off-diagonal 128 x 128 block of its decay mask enters
// through the state at the chunk's midpoint, which is that block's exact rank-N
// factorisation.  After the per-block decay cumsum (prefill_simt.cu) come two kernels:
//
// chunk_state_walk_kernel -- persistent: one CTA per (batch b, group g, 1-3 heads) walks
//   the blocks of its heads in order, the carried state held in the state warps'
//   registers (no cross-CTA hand-off):
//     S_k = B_k^T (w o X_k),  w_s = exp(Lam_end - Lam_s) dt_s         (tcgen05, fp16 in)
//     H_{k+1} = exp(Lam_end) H_k + S_k                                 (fp32)
//   and writes every block's start state H_k once, as the bf16 operand image the output
//   kernel loads, plus the final state.
//
// block_output_kernel -- one CTA per (block k, range of heads of one group, b),
//   warp-specialised: warp 0 issues TMA and bulk loads, warp 1 issues tcgen05.mma, warps
//   4-11 build the masked matrix P in TMEM, warps 12-15 run the epilogue:
//     G  = C_k B_k^T                            (once per CTA; shared by its heads)
//     P  = G o exp(Lam_t - Lam_s) o dt_s (s <= t), bf16 in TMEM (the MMA's A operand)
//     Yd = P X,  Yo = C_k H_k^T                 (tcgen05)
//     y  = Yd + exp(Lam_t) Yo + D_h x_t  -> bf16
//
// Both kernels are launched as programmatic dependents: their setup (barriers, TMEM, and
// for the output kernel the C/B loads and G) overlaps the previous kernel's tail.  Every
// wait is bounded; expiry records SSD_ERR_TIMEOUT in the device error word and the CTA
// drains without further waiting.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "prefill_tc.h"
#include "ptx.cuh"

namespace ssd {

using namespace ptx;

namespace {

constexpr int kBox = 16384;                    // one TMA box: 128 rows x 128 bytes
constexpr int kHImage = 16384;                 // bf16 H_c image: 2 x 64 rows x 128 B
constexpr int kBlk = 128;                       // tokens per block of the tensor-core path
constexpr int kP = 64, kN = 128;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ================================================================ packed variable-length table
// From cu_seqlens (nseq + 1 token offsets): the first Q-token block of every sequence (the
// exclusive prefix sum of ceil(len / Q)), then the total, and the sequence of every block
// (-1 past the total).  Offsets that do not start at 0, decrease, or do not end at
// total_tokens record SSD_ERR_SHAPE and leave every block empty (no kernel then does work).
constexpr int kTableThreads = 1024;

__global__ void __launch_bounds__(kTableThreads)
varlen_table_kernel(const int* __restrict__ cu, int nseq, int total_tokens, int max_blocks, int Q,
                    int* __restrict__ first, int* __restrict__ seqof, int* err)
{
    __shared__ int part[kTableThreads];
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0) bad = (cu[0] != 0 || cu[nseq] != total_tokens) ? 1 : 0;
    __syncthreads();
    const int per = (nseq + kTableThreads - 1) / kTableThreads;
    const int s0 = min(nseq, tid * per), s1 = min(nseq, s0 + per);
    int sum = 0, neg = 0;
    for (int s = s0; s < s1; ++s) {
        const int len = cu[s + 1] - cu[s];
        neg |= len < 0;
        sum += (max(len, 0) + Q - 1) / Q;
    }
    if (neg) atomicOr(&bad, 1);
    part[tid] = sum;
    __syncthreads();
    for (int o = 1; o < kTableThreads; o <<= 1) {      // inclusive scan of the partial counts
        const int v = tid >= o ? part[tid - o] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    const int total = part[kTableThreads - 1];
    if (bad || total > max_blocks) {
        if (tid == 0) record_error(err, SSD_ERR_SHAPE);
        for (int i = tid; i < max_blocks; i += kTableThreads) seqof[i] = -1;
        for (int i = tid; i <= nseq; i += kTableThreads) first[i] = 0;
        return;
    }
    int base = tid ? part[tid - 1] : 0;
    for (int s = s0; s < s1; ++s) {
        first[s] = base;
        const int nb = (cu[s + 1] - cu[s] + Q - 1) / Q;
        for (int k = 0; k < nb; ++k) seqof[base + k] = s;
        base += nb;
    }
    if (tid == 0) first[nseq] = total;
    for (int i = total + tid; i < max_blocks; i += kTableThreads) seqof[i] = -1;
}

// ================================================================ chunk states: persistent walk
// One resident CTA per (batch b, group g, range of 1-3 heads) walks the chunks of its
// heads in order, so the carried state never leaves the CTA (registers) and no chunk
// waits for another CTA.  The heads' chunk states form one tcgen05 chain with the heads
// stacked along N (N = 64 x heads); B_c is staged once per chunk for all of them.
// Operands stream through a ring of 64-row stages, three deep with one head per CTA and
// four with up to three (fp16 B rows, one X box per head, the heads' weights w_s); two
// TMEM accumulators alternate between chunks.  Warp-specialised: one warp issues the
// loads, one the MMAs, four warps form X~ = w o X, and eight state warps (which hold the
// carried state) update it as soon as a chunk's accumulator is complete and hand the
// accumulator back, so that the update overlaps the conversion of the next stages.  Each
// state warp writes its own 2 KB piece of every bf16 start-state image (the image's
// 64-byte-swizzled layout makes that piece contiguous) and stores it with one bulk copy,
// so the update needs no CTA-wide barrier.  The block decay comes from the weights rows
// in global memory, read a block ahead.
constexpr int kWalkWorkers = 8;                               // state warps w, w + 4: TMEM lane quarter w
constexpr int kWalkConv = 4;                                  // warps forming X~ = w o X
constexpr int kWalkThreads = (kWalkWorkers + 2 + kWalkConv) * 32;   // + load warp + MMA warp
constexpr int kQBox = 8192;                                   // one 64-row x 128-byte box
constexpr int kWRow = 68;                                     // weights per head in a stage (+ decay)

// Two shapes of the walk: up to three heads per CTA, one CTA per SM (many chains per SM);
// or one head per CTA with two CTAs per SM, so that two latency-bound chains interleave
// (when all chains fit in two CTAs per SM).
template <int NH>
struct WalkCfg {
    static constexpr int kStages = NH == 1 ? 3 : 4;
    static constexpr int kCtasPerSm = NH == 1 ? 2 : 1;
    static constexpr uint32_t kTmemCols = NH == 1 ? 128 : 512;     // two accumulators of 64 NH columns
    static constexpr uint32_t kAccStride = NH == 1 ? 64 : 256;
    static constexpr int kStageX = 2 * kQBox;                       // after the B rows
    static constexpr int kStageW = kStageX + NH * kQBox;            // float[heads][68]
    static constexpr int kStageBytes = kStageW + 1024;
    static constexpr int kImg = kStages * kStageBytes;              // state images, one per head
    static constexpr int kBar = kImg + NH * kHImage;                // full, conv, empty, acc, acc free
    static constexpr int kSlot = kBar + (3 * kStages + 4) * 8;
    static constexpr int kBytes = kSlot + 16 + 1024;
    static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
    static_assert(kBytes * kCtasPerSm <= 227 * 1024, "walk shared memory");
};

struct WalkMaps {
    CUtensorMap x1, x2;          // x as (P, T, H, b), boxes of 1 / 2 heads x 64 rows
    CUtensorMap b;               // fp16 B as (64, T, 2G, b), box: both halves x 64 rows
    CUtensorMap w;               // weights as (nchunks (Q + 4), b H) fp32, box 68 x 3 heads
};

template <int Q, int NH>
__global__ void __launch_bounds__(kWalkThreads, WalkCfg<NH>::kCtasPerSm)
chunk_state_walk_kernel(const __grid_constant__ WalkMaps maps, const float* __restrict__ wts,
                        const float* __restrict__ init_state, float* final_state,
                        uint8_t* __restrict__ himg, int nheads, int ngroups, int nchunks,
                        int ctas_per_group, int* err, const int* __restrict__ vl_cu,
                        const int* __restrict__ vl_first)
{
    using L = WalkCfg<NH>;
    constexpr int NQ = Q / 64;                          // stages per chunk
    constexpr int S = L::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* conv = full + S;
    uint64_t* empty = conv + S;
    uint64_t* accb = empty + S;
    uint64_t* accfree = accb + 2;
    uint32_t* slot = reinterpret_cast<uint32_t*>(sm + L::kSlot);

    // this CTA's heads: a contiguous range of one (b, g)
    const int hpg = nheads / ngroups;
    const int unit = blockIdx.x / ctas_per_group, part = blockIdx.x - unit * ctas_per_group;
    const int b = unit / ngroups, g = unit - b * ngroups;
    const int hlo = g * hpg + (part * hpg) / ctas_per_group;
    const int nh = g * hpg + ((part + 1) * hpg) / ctas_per_group - hlo;     // 1..3
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the chain's blocks: batched, chunks 0 .. nchunks - 1 of batch b; packed variable-length
    // (b is then the sequence), the sequence's blocks blk0 .. blk0 + nblk - 1, whose rows
    // start at row0 of the single batch
    int row0 = 0, blk0 = 0, nblk = nchunks, bt = b;
    if (vl_first) {
        griddep_wait();                                  // the block table comes from an earlier kernel
        row0 = vl_cu[b];
        blk0 = vl_first[b];
        nblk = vl_first[b + 1] - blk0;
        bt = 0;
    }
    const int sb = vl_first ? 0 : b;                     // batch index of the per-block arrays
    const int total = nblk * NQ;
    auto stage = [&](int st) { return sm + st * L::kStageBytes; };

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&conv[i], kWalkConv);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accb[i], 1);
            mbar_init(&accfree[i], kWalkWorkers);
        }
        fence_mbar_init();
    }
    if (warp == kWalkWorkers + 1) {
        tmem_alloc(slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    griddep_launch_dependents();

    if (warp == kWalkWorkers) {
        // ---------------------------------------------------------------- loads
        if (lane == 0) {
            griddep_wait();                              // fp16 B and the weights come from the cumsum kernel
            int issued = 0;
            for (int k = 0; k < total; ++k) {
                const int st = k % S;
                if (k >= S && !mbar_wait(&empty[st], ((k / S) + 1) & 1, err)) break;
                const int c = k / NQ, qq = k - c * NQ, row = row0 + c * Q + qq * 64;
                uint8_t* sg = stage(st);
                mbar_expect_tx(&full[st], (2 + nh) * kQBox + NH * kWRow * 4);
                tma_load_4d(sg, &maps.b, 0, row, 2 * g, bt, &full[st]);
                int hh = 0;
                if (NH > 1 && nh >= 2) {
                    tma_load_4d(sg + L::kStageX + hh * kQBox, &maps.x2, 0, row, hlo + hh, bt, &full[st]);
                    hh += 2;
                }
                if (nh - hh >= 1)
                    tma_load_4d(sg + L::kStageX + hh * kQBox, &maps.x1, 0, row, hlo + hh, bt, &full[st]);
                tma_load_2d(sg + L::kStageW, &maps.w, (blk0 + c) * (Q + 4) + qq * 64, sb * nheads + hlo, &full[st]);
                issued = k + 1;
            }
            // the CTA does not exit with loads in flight
            for (int k = max(0, issued - S); k < issued; ++k) mbar_wait(&full[k % S], (k / S) & 1, err);
        }
    } else if (warp == kWalkWorkers + 1) {
        // ---------------------------------------------------------------- MMAs
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(128, 64 * nh, true, true);
            int done = 0;
            for (int k = 0; k < total; ++k) {
                const int st = k % S, c = k / NQ, qq = k - c * NQ;
                if (!mbar_wait(&conv[st], (k / S) & 1, err)) break;
                // the state warps have read this accumulator's previous block (c - 2)
                if (qq == 0 && c >= 2 && !mbar_wait(&accfree[c & 1], ((c >> 1) - 1) & 1, err)) break;
                tc_fence_after();
                const uint32_t aB = smem_u32(stage(st)), aX = aB + L::kStageX;
                // S_c[n][64 hh + p] += sum_s B_s[n] X~_s[hh][p] over this stage's 64 rows
                const uint64_t dB = smem_desc_sw128(aB, kQBox, 1024), dX = smem_desc_sw128(aX, kQBox, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_f16(tmem + (c & 1) * L::kAccStride, desc_advance(dB, ks * 2048), desc_advance(dX, ks * 2048),
                             idesc, (qq > 0 || ks > 0) ? 1u : 0u);
                umma_commit(&empty[st]);
                if (qq == NQ - 1) umma_commit(&accb[c & 1]);
                done = k + 1;
            }
            // the CTA does not release TMEM with MMAs in flight
            if (done > 0) mbar_wait(&empty[(done - 1) % S], ((done - 1) / S) & 1, err);
        }
    } else if (warp >= kWalkWorkers + 2) {
        // ---------------------------------------------------------------- X~ = w o X (fp16)
        // consecutive threads take consecutive 16-byte chunks; chunk i: head i / 512, row
        // (i / 8) % 64
        const int ctid = tid - (kWalkWorkers + 2) * 32;
        for (int k = 0; k < total; ++k) {
            const int st = k % S;
            if (!mbar_wait(&full[st], (k / S) & 1, err)) break;
            uint4* sx = reinterpret_cast<uint4*>(stage(st) + L::kStageX);
            const float* sw = reinterpret_cast<const float*>(stage(st) + L::kStageW);
            constexpr int kPer = NH * 512 / (kWalkConv * 32);                 // chunks per thread
            constexpr int kBatch = kPer % 3 == 0 ? 3 : kPer;                  // loads in flight
            static_assert(kPer % kBatch == 0, "conversion batches");
#pragma unroll
            for (int j0 = 0; j0 < kPer; j0 += kBatch) {
                uint4 u[kBatch];
                float w[kBatch];
#pragma unroll
                for (int j = 0; j < kBatch; ++j) {
                    const int i = ctid + (j0 + j) * kWalkConv * 32;
                    if (i < nh * 512) {
                        u[j] = sx[i];
                        w[j] = sw[(i >> 9) * kWRow + ((i >> 3) & 63)];
                    }
                }
#pragma unroll
                for (int j = 0; j < kBatch; ++j) {
                    const int i = ctid + (j0 + j) * kWalkConv * 32;
                    if (i < nh * 512) {
                        uint4 v = u[j];
                        v.x = pack_f16x2(bf16lo(v.x) * w[j], bf16hi(v.x) * w[j]);
                        v.y = pack_f16x2(bf16lo(v.y) * w[j], bf16hi(v.y) * w[j]);
                        v.z = pack_f16x2(bf16lo(v.z) * w[j], bf16hi(v.z) * w[j]);
                        v.w = pack_f16x2(bf16lo(v.w) * w[j], bf16hi(v.w) * w[j]);
                        sx[i] = v;
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[st]);
        }
    } else {
        // ---------------------------------------------------------------- state warps
        // carried state: thread owns column n and rows p = 32 half + pp, for each head; the
        // update of block c runs as soon as its accumulator is complete, while the converter
        // warps already form the next stages
        const int n = (warp & 3) * 32 + lane;
        const int half = warp >> 2;
        float Hs[NH][32];
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) {
                const int p = half * 32 + pp;
                Hs[hh][pp] = (hh < nh && init_state)
                                 ? init_state[((size_t)(b * nheads + hlo + hh) * kP + p) * kN + n] : 0.f;
            }
        }
        bool ok = true;
        // block decay exp(Lam_end) of each head, read from the weights rows a block ahead
        const size_t wrow = (size_t)nchunks * (Q + 4);
        const float* wlast = wts + (size_t)(sb * nheads + hlo) * wrow + Q;
        auto load_e = [&](int c, float (&e)[NH]) {
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) e[hh] = hh < nh ? wlast[hh * wrow + (size_t)(blk0 + c) * (Q + 4)] : 0.f;
        };

        // bf16 image of the carried state as the start state of chunk cc.  The image is the
        // MN-major operand tile with 64-byte swizzle: two p-halves of [128 n][32 p], row n of
        // a half holding p in four 16-byte chunks, chunk j stored at j ^ ((n / 2) mod 4).
        // This warp's piece (rows 32 (warp mod 4) .. + 31 of half warp / 4) is contiguous.
        const uint32_t piece = half * 8192 + (warp & 3) * 2048;
        auto write_images = [&](int cc) {
            if (lane == 0) bulk_wait_group_read0();      // this warp's previous stores have read
            __syncwarp();
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
                if (hh < nh) {
                    uint8_t* row = sm + L::kImg + hh * kHImage + piece + lane * 64;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const float* h8 = &Hs[hh][8 * jj];
                        *reinterpret_cast<uint4*>(row + ((jj ^ ((n >> 1) & 3)) << 4)) =
                            make_uint4(pack_bf16x2(h8[0], h8[1]), pack_bf16x2(h8[2], h8[3]),
                                       pack_bf16x2(h8[4], h8[5]), pack_bf16x2(h8[6], h8[7]));
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                for (int hh = 0; hh < nh; ++hh)
                    bulk_store(himg + ((size_t)(sb * nheads + hlo + hh) * nchunks + blk0 + cc) * kHImage + piece,
                               sm + L::kImg + hh * kHImage + piece, 2048);
                bulk_commit_group();
            }
        };

        if (nblk > 0) write_images(0);
        float e_next[NH];
        griddep_wait();                                  // the weights rows come from the cumsum kernel
        if (nblk > 0) load_e(0, e_next);
        for (int c = 0; c < nblk && ok; ++c) {
            float e[NH];
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) e[hh] = e_next[hh];
            if (c + 1 < nblk) load_e(c + 1, e_next);
            // H <- exp(Lam_end) H + S_c: the start state of block c + 1
            ok = mbar_wait(&accb[c & 1], (c >> 1) & 1, err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t acc = tmem + (c & 1) * L::kAccStride + ((uint32_t)((warp & 3) * 32) << 16) + half * 32;
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
                if (hh < nh) {                           // uniform across the CTA
#pragma unroll
                    for (int q16 = 0; q16 < 2; ++q16) {
                        uint32_t v[16];
                        tmem_ld16(acc + hh * 64 + 16 * q16, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            Hs[hh][16 * q16 + j] = fmaf(e[hh], Hs[hh][16 * q16 + j], __uint_as_float(v[j]));
                    }
                }
            }
            // the accumulator may take block c + 2
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accfree[c & 1]);
            if (c + 1 < nblk) write_images(c + 1);
        }
        if (lane == 0) bulk_wait_group0();
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
            if (hh < nh) {
#pragma unroll
                for (int pp = 0; pp < 32; ++pp) {
                    const int p = half * 32 + pp;
                    final_state[((size_t)(b * nheads + hlo + hh) * kP + p) * kN + n] = Hs[hh][pp];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWalkWorkers + 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}



// ================================================================ block output
// One CTA per (128-token block k, head group, batch b); warp 0 issues TMA and bulk loads,
// warp 1 issues tcgen05.mma, warps 4-11 build the masked diagonal operand, warps 12-15
// run the epilogue.  With t, s the block's tokens and Lam the decay cumsum from the
// block start:
//
//   G   = C_t B_s^T                           (once per CTA; fp32 in TMEM, shared by the heads)
//   per head h (operand slots three deep, P buffers and accumulators double/triple-buffered):
//     P   = G o exp(Lam_t - Lam_s) o dt_s     (s <= t; bf16)
//     Yd  = P X_s,   Yo = C_t H_k^T           (tcgen05; H_k = state at the block start)
//     y_t = Yd + exp(Lam_t) Yo + D_h x_t      -> bf16, written over x_t and TMA-stored
//
// A chunk longer than 128 tokens is handled as consecutive 128-token blocks: its strictly
// lower off-diagonal blocks enter through the state at each block start (the exact rank-N
// factorisation of those blocks), which the chunk-state walk provides every 128 tokens.
// Below-diagonal 32-column sub-blocks of P use exp(Lam_t - Lam_q) exp(Lam_q - Lam_s) with q
// the sub-block's last column (both <= 1); sub-blocks on the diagonal use the first column
// as reference when their own decay is below 40 (both factors within e^+-40) and fall
// back to one exponential per element otherwise.
constexpr int kOutThreads = 512;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpP0 = 4, kWarpE0 = 12;
constexpr int kPThreads = 256, kEThreads = 128;
constexpr int kXSlots = 6;                               // x / y operand slots
constexpr int kHSlots = 3;                               // state image slots (freed after Yo)
constexpr int kAccSlots = 3;                             // TMEM accumulator pairs
constexpr uint32_t kColG = 384;                          // TMEM columns of G, later of the two P buffers
constexpr uint32_t kAccCols = 128;                       // per accumulator: Yd +0, Yo +64

struct OutSmem {
    static constexpr int kC = 0;                         // C_t [2 n-halves][128 rows][128 B]
    static constexpr int kB = 2 * kBox;                  // B_s (operand of G)
    static constexpr int kH0 = kB + 2 * kBox;            // state image slots (MN-major, 16 KB each)
    static constexpr int kSlot0 = kH0 + kHSlots * kHImage;  // x slots
    static constexpr int kXo = 0;                        //   x (then y) [128 rows][128 B]
    static constexpr int kLo = kBox;                     //   Lam[128]
    static constexpr int kDo = kLo + 512;                //   dt[128]
    static constexpr int kVo = kDo + 512;                //   column factors, sub-block-end reference
    static constexpr int kWo = kVo + 512;                //   column factors, sub-block-start reference
    static constexpr int kSlotBytes = (kWo + 512 + 1023) / 1024 * 1024;
    static constexpr int kBar = kSlot0 + kXSlots * kSlotBytes;
    static constexpr int kNumBars = 2 + 2 * kXSlots + 2 * kAccSlots + kHSlots + 4;
    static constexpr int kSlotTm = kBar + kNumBars * 8;
    static constexpr int kAbort = kSlotTm + 4;
    static constexpr int kBytes = kAbort + 12 + 1024;
};
static_assert(OutSmem::kSlotBytes % 1024 == 0, "slots keep 1024-byte alignment");
static_assert(OutSmem::kBytes <= 227 * 1024, "output shared memory");

enum { BAR_CB = 0, BAR_S = 1, BAR_XFULL = 2, BAR_XEMPTY = BAR_XFULL + kXSlots,
       BAR_AFULL = BAR_XEMPTY + kXSlots, BAR_AEMPTY = BAR_AFULL + kAccSlots,
       BAR_HEMPTY = BAR_AEMPTY + kAccSlots, BAR_PFULL = BAR_HEMPTY + kHSlots, BAR_PEMPTY = BAR_PFULL + 2 };

__global__ void __launch_bounds__(kOutThreads, 1)
block_output_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                    const float* __restrict__ fac,
                    const uint8_t* __restrict__ himg, const float* __restrict__ D, int nheads,
                    int ngroups, int nblocks, int heads_per_cta, int* err, __nv_bfloat16* __restrict__ y,
                    const int* __restrict__ vl_cu, const int* __restrict__ vl_first,
                    const int* __restrict__ vl_seq)
{
    using L = OutSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint8_t* sC = sm + L::kC;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kSlotTm);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kAbort);

    // block k: rows t0 .. t0 + 127 of batch b; in packed variable-length mode (batch 1) block k
    // of the table, rows t0 .. t0 + len - 1 of its sequence (the rest belong to the next one:
    // their dt is 0, and their y rows are not stored)
    const int k = blockIdx.x, hg = blockIdx.y;
    int b = blockIdx.z, t0 = k * kBlk, len = kBlk;
    if (vl_seq) {
        int sq;
        if (!varlen_block(vl_cu, vl_first, vl_seq, k, kBlk, &sq, &t0, &len)) return;
        b = 0;
    }
    const int h0 = hg * heads_per_cta;
    const int g = h0 / (nheads / ngroups);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        mbar_init(&bars[BAR_CB], 1);
        mbar_init(&bars[BAR_S], 1);
        for (int s = 0; s < kXSlots; ++s) {
            mbar_init(&bars[BAR_XFULL + s], 1);
            mbar_init(&bars[BAR_XEMPTY + s], 1);
        }
        for (int s = 0; s < kAccSlots; ++s) {
            mbar_init(&bars[BAR_AFULL + s], 1);
            mbar_init(&bars[BAR_AEMPTY + s], kEThreads);
        }
        for (int s = 0; s < kHSlots; ++s) mbar_init(&bars[BAR_HEMPTY + s], 1);
        for (int p = 0; p < 2; ++p) {
            mbar_init(&bars[BAR_PFULL + p], kPThreads);
            mbar_init(&bars[BAR_PEMPTY + p], 1);
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

    auto slot = [&](int s) { return sm + L::kSlot0 + s * L::kSlotBytes; };
    auto hslot = [&](int s) { return sm + L::kH0 + s * kHImage; };
    // P buffer p: 64 TMEM columns (128 bf16 per row), over G's columns once G is in registers
    auto pcol = [&](int p) { return kColG + (uint32_t)p * 64; };

    if (warp == kWarpTma) {
        if (lane == 0) {
            mbar_expect_tx(&bars[BAR_CB], 4 * kBox);
            tma_load_3d(sC, &tm_c, g * kN, t0, b, &bars[BAR_CB]);
            tma_load_3d(sC + kBox, &tm_c, g * kN + 64, t0, b, &bars[BAR_CB]);
            tma_load_3d(sm + L::kB, &tm_b, g * kN, t0, b, &bars[BAR_CB]);
            tma_load_3d(sm + L::kB + kBox, &tm_b, g * kN + 64, t0, b, &bars[BAR_CB]);
            griddep_wait();                              // block factors and state images come from earlier kernels
            for (int j = 0; j < heads_per_cta; ++j) {
                const int s = j % kXSlots, hs = j % kHSlots;
                const size_t bh = (size_t)b * nheads + h0 + j;
                if (j >= kXSlots &&
                    !mbar_wait_or_abort(&bars[BAR_XEMPTY + s], (j / kXSlots - 1) & 1, err, abort_flag))
                    break;
                if (j >= kHSlots &&
                    !mbar_wait_or_abort(&bars[BAR_HEMPTY + hs], (j / kHSlots - 1) & 1, err, abort_flag))
                    break;
                uint8_t* sl = slot(s);
                mbar_expect_tx(&bars[BAR_XFULL + s], kBox + kHImage + 4 * 512);
                tma_load_3d(sl + L::kXo, &tm_x, (h0 + j) * kP, t0, b, &bars[BAR_XFULL + s]);
                bulk_load(hslot(hs), himg + (bh * nblocks + k) * kHImage, kHImage, &bars[BAR_XFULL + s]);
                bulk_load(sl + L::kLo, fac + (bh * nblocks + k) * 4 * kBlk, 4 * 512, &bars[BAR_XFULL + s]);
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0 && mbar_wait_or_abort(&bars[BAR_CB], 0, err, abort_flag)) {
            tc_fence_after();
            const uint32_t aC = smem_u32(sC), aB = smem_u32(sm + L::kB);
            // G = C_t B_s^T (K = N = 128 state columns) into columns [384, 512)
            const uint32_t idG = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kb = ks >> 2, off = (ks & 3) * 32;
                umma_f16(tmem + kColG, smem_desc_sw128(aC + kb * kBox + off, 16, 1024),
                         smem_desc_sw128(aB + kb * kBox + off, 16, 1024), idG, ks > 0 ? 1u : 0u);
            }
            umma_commit(&bars[BAR_S]);
            constexpr uint32_t idMN = idesc_bf16_f32(128, 64, false, true);
            const uint64_t dC = smem_desc_sw128(aC, 16, 1024);
            // Yo of a head is issued as soon as its slot is loaded (and its accumulator free),
            // Yd as soon as its P is built; the two streams are polled, not ordered
            int jo = 0, jd = 0;
            uint32_t idle = 0;
            while (jd < heads_per_cta) {
                bool progressed = false;
                if (jo < heads_per_cta) {
                    const int s = jo % kXSlots, a = jo % kAccSlots;
                    if (mbar_test_wait(&bars[BAR_XFULL + s], (jo / kXSlots) & 1) &&
                        (jo < kAccSlots || mbar_test_wait(&bars[BAR_AEMPTY + a], (jo / kAccSlots - 1) & 1))) {
                        tc_fence_after();
                        const uint32_t aH = smem_u32(hslot(jo % kHSlots));
                        // Yo = C_t H_k^T: A = C (K-major over n), B = H image (MN-major, 64-byte
                        // swizzle: p-halves 8 KB apart, 8-row groups of n 512 B apart)
                        const uint64_t dH = smem_desc_sw64(aH, 8192, 512);
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            const uint32_t kb = ks >> 2, off = (ks & 3) * 32;
                            umma_f16(tmem + a * kAccCols + 64, desc_advance(dC, kb * kBox + off),
                                     desc_advance(dH, ks * 1024), idMN, ks > 0 ? 1u : 0u);
                        }
                        umma_commit(&bars[BAR_HEMPTY + jo % kHSlots]);
                        ++jo;
                        progressed = true;
                    }
                }
                if (jd < jo) {
                    const int s = jd % kXSlots, a = jd % kAccSlots, p = jd & 1;
                    if (mbar_test_wait(&bars[BAR_PFULL + p], (jd >> 1) & 1)) {
                        tc_fence_after();
                        const uint64_t dX = smem_desc_sw128(smem_u32(slot(s) + L::kXo), kBox, 1024);
                        // Yd = P X: A = P in TMEM (eight columns per 16 tokens), B = X (MN-major)
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            umma_f16_ts(tmem + a * kAccCols, tmem + pcol(p) + ks * 8, desc_advance(dX, ks * 2048),
                                        idMN, ks > 0 ? 1u : 0u);
                        umma_commit(&bars[BAR_PEMPTY + p]);
                        umma_commit(&bars[BAR_AFULL + a]);
                        ++jd;
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
        }
    } else if (warp >= kWarpP0 && warp < kWarpE0) {
        const int pw = warp - kWarpP0;
        const int q = warp & 3, colhalf = pw >> 2;
        const int r = q * 32 + lane;                    // block row t
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        bool live = mbar_wait_or_abort(&bars[BAR_S], 0, err, abort_flag);
        tc_fence_after();
        // this thread's G entries (row r, sub-blocks kc0 and kc1), the same for every head;
        // once every P thread holds its entries, G's columns become the P buffers
        const int kc0 = colhalf, kc1 = colhalf + 2;
        uint32_t v0[32], v1[32];
        tmem_ld32(trow + kColG + kc0 * 32, v0);
        tmem_ld32(trow + kColG + kc1 * 32, v1);
        tmem_wait_ld();
        tc_fence_before();
        live = named_bar_and(1, kPThreads, live);
        tc_fence_after();
        // Every thread waits on the barriers itself (bounded), so the loop needs no
        // named barrier; a thread that gives up leaves PFULL incomplete and the MMA
        // thread's bounded wait reports it.
        for (int j = 0; j < heads_per_cta && live; ++j) {
            const int s = j % kXSlots, p = j & 1;
            live = mbar_wait_or_abort(&bars[BAR_XFULL + s], (j / kXSlots) & 1, err, abort_flag) &&
                   // the GEMM of head j - 2 must be done with this P buffer
                   (j < 2 || mbar_wait_or_abort(&bars[BAR_PEMPTY + p], ((j >> 1) - 1) & 1, err, abort_flag));
            if (!live) break;
            uint8_t* sl = slot(s);
            // Lam, dt and the column factors of each 32-column sub-block: sV references the
            // sub-block's last column (factor <= 1), sW its first (used only where the
            // sub-block's own decay is small)
            const float* sLam = reinterpret_cast<const float*>(sl + L::kLo);
            const float* sDt = reinterpret_cast<const float*>(sl + L::kDo);
            const float* sV = reinterpret_cast<const float*>(sl + L::kVo);
            const float* sW = reinterpret_cast<const float*>(sl + L::kWo);
            const float lam_t = sLam[r];
#pragma unroll
            for (int w2 = 0; w2 < 2; ++w2) {
                const int kc = w2 ? kc1 : kc0;
                const uint32_t* v = w2 ? v1 : v0;
                const int s0 = kc * 32;
                uint32_t pk[16];
                // the branch is taken by the warp's 32 rows (q * 32 ..) alike: a diagonal
                // sub-block is one path for the whole warp, not two in series
                if (kc < q) {
                    const float u = expf(lam_t - sLam[s0 + 31]);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * u * sV[s0 + 2 * e],
                                            __uint_as_float(v[2 * e + 1]) * u * sV[s0 + 2 * e + 1]);
                } else if (kc > q) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                } else if (sLam[s0] - sLam[s0 + 31] < 40.f) {
                    // sub-block on the diagonal with modest internal decay:
                    // exp(Lam_t - Lam_s) = exp(Lam_t - Lam_s0) exp(Lam_s0 - Lam_s), both
                    // factors within e^+-40 (fully normal fp32)
                    const float u = expf(lam_t - sLam[s0]);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int sa = s0 + 2 * e;
                        const float pa = __uint_as_float(v[2 * e]) * u * sW[sa];
                        const float pb = __uint_as_float(v[2 * e + 1]) * u * sW[sa + 1];
                        pk[e] = pack_bf16x2(sa <= r ? pa : 0.f, sa + 1 <= r ? pb : 0.f);
                    }
                } else {
                    // strong decay inside the sub-block: one exponential per element
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int sa = s0 + 2 * e, sb = sa + 1;
                        const float pa = sa <= r ? __uint_as_float(v[2 * e]) * expf(lam_t - sLam[sa]) * sDt[sa] : 0.f;
                        const float pb = sb <= r ? __uint_as_float(v[2 * e + 1]) * expf(lam_t - sLam[sb]) * sDt[sb] : 0.f;
                        pk[e] = pack_bf16x2(pa, pb);
                    }
                }
                tmem_st16(trow + pcol(p) + kc * 16, pk);  // tokens 32 kc .. 32 kc + 31 of row r
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[BAR_PFULL + p]);
        }
    } else if (warp >= kWarpE0) {
        // ---- epilogue: y = Yd + exp(Lam_t) Yo + D x, written in place over the block's
        // x rows (each thread its own row), then one TMA store of the block
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const int etid = tid - kWarpE0 * 32;
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        for (int j = 0; j < heads_per_cta; ++j) {
            const int s = j % kXSlots, a = j % kAccSlots;
            if (!mbar_wait_or_abort(&bars[BAR_AFULL + a], (j / kAccSlots) & 1, err, abort_flag)) break;
            tc_fence_after();
            const int h = h0 + j;
            uint8_t* sl = slot(s);
            const float u = expf(reinterpret_cast<const float*>(sl + L::kLo)[r]);
            const float Dh = D[h];
            uint8_t* xrow = sl + L::kXo + r * 128;
            const uint32_t acc = trow + a * kAccCols;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t yd[32], yo[32];
                tmem_ld32(acc + half * 32, yd);
                tmem_ld32(acc + 64 + half * 32, yo);
                tmem_wait_ld();
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int qx = half * 4 + qq;
                    uint4* xp = reinterpret_cast<uint4*>(xrow + ((qx ^ (r & 7)) << 4));
                    const uint4 xu = *xp;
                    const uint32_t xw[4] = {xu.x, xu.y, xu.z, xu.w};
                    uint32_t o[4];
#pragma unroll
                    for (int k2 = 0; k2 < 4; ++k2) {
                        const int jj = qq * 8 + 2 * k2;
                        const float a0 = fmaf(u, __uint_as_float(yo[jj]), __uint_as_float(yd[jj])) + Dh * bf16lo(xw[k2]);
                        const float a1 = fmaf(u, __uint_as_float(yo[jj + 1]), __uint_as_float(yd[jj + 1])) + Dh * bf16hi(xw[k2]);
                        o[k2] = pack_bf16x2(a0, a1);
                    }
                    if (len == kBlk)
                        *xp = make_uint4(o[0], o[1], o[2], o[3]);
                    else if (r < len)                       // partial block: the row goes out directly
                        *reinterpret_cast<uint4*>(y + ((size_t)(t0 + r) * nheads + h) * kP + qx * 8) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[BAR_AEMPTY + a]);
            fence_proxy_async_smem();                       // y rows -> visible to the TMA unit
            named_bar_sync(2, kEThreads);
            if (etid == 0) {
                if (len == kBlk) {
                    tma_store_3d(&tm_y, h * kP, t0, b, sl + L::kXo);
                    bulk_commit_group();
                    bulk_wait_group_read0();                // the slot may be refilled now
                }
                mbar_arrive(&bars[BAR_XEMPTY + s]);
            }
        }
        if (etid == 0) bulk_wait_group0();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
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

// 16-bit tensor [outer][rows][inner] read in boxes of 64 (inner) x box_rows, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
              CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint32_t box_rows = 128)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, rows, outer};
    cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, type, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled map of `rank` dimensions (dim 0 contiguous; strides in bytes for dims 1..rank-1),
// 128-byte swizzle or none; out-of-range elements read as zero.
bool encode_map(CUtensorMap* m, CUtensorMapDataType type, int rank, const void* base,
                const uint64_t* dims, const uint64_t* strides, const uint32_t* box, bool swizzle)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i) gs[i - 1] = strides[i - 1];
    }
    return fn(m, type, rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count();

// Heads per output CTA: a divisor of the heads per group (so a CTA's heads share one B/C
// group), chosen to minimise waves x (heads + 3): each CTA pays about three heads' worth
// of pipeline fill and drain, and G = C B^T is computed once per CTA.
int heads_per_cta(const Dims& d)
{
    const int hpg = d.nheads / d.ngroups;
    const long long units = (long long)d.nchunks * d.batch * d.ngroups;     // (block, b, g)
    const int sms = sm_count();
    int best = 1;
    long long best_cost = -1;
    for (int k = 1; k <= hpg && k <= 64; ++k) {
        if (hpg % k) continue;
        const long long ctas = units * (hpg / k);
        const long long cost = (ctas + sms - 1) / sms * (k + 3);
        if (best_cost < 0 || cost < best_cost || (cost == best_cost && k > best)) {
            best = k;
            best_cost = cost;
        }
    }
    return best;
}

int sm_count()
{
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev] && cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        cache[dev] = 148;
    return cache[dev];
}

// Walk shape: one head per CTA (two CTAs per SM) when every (b, h) chain fits in the
// SMs that way, else up to three heads per CTA.
// (b, h) chains of the walk: batch x heads, or sequences x heads in packed variable-length mode
long long walk_chains(const Dims& d) { return (long long)(d.nseq ? d.nseq : d.batch) * d.nheads; }

int walk_heads(const Dims& d)
{
    return walk_chains(d) <= (long long)WalkCfg<1>::kCtasPerSm * sm_count() ? 1 : 3;
}

// CTAs per (b, g) of the walk: enough that each holds at most nh heads, and as many as
// fill the SMs otherwise (never more than there are heads).
int walk_ctas_per_group(const Dims& d, int nh)
{
    const int hpg = d.nheads / d.ngroups;
    const int units = (d.nseq ? d.nseq : d.batch) * d.ngroups;
    int cpg = (hpg + nh - 1) / nh;
    cpg = max(cpg, sm_count() / units);
    return min(cpg, hpg);
}

template <int Q, int NH>
cudaError_t walk_t(const Dims& d, const WalkMaps& maps, const TcWorkspace& w, const float* init_state,
                   float* final_state, cudaStream_t s)
{
    auto k = chunk_state_walk_kernel<Q, NH>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         WalkCfg<NH>::kBytes);
    if (e != cudaSuccess) return e;
    const int cpg = walk_ctas_per_group(d, NH);
    const unsigned grid = (unsigned)((d.nseq ? d.nseq : d.batch) * d.ngroups * cpg);
    return launch_dependent(k, dim3(grid), dim3(kWalkThreads), WalkCfg<NH>::kBytes, s, maps,
                            static_cast<const float*>(w.wts),
                            init_state, final_state, w.himg, d.nheads, d.ngroups, d.nchunks, cpg,
                            device_error_word(), d.cu_seqlens, d.vl_first);
}

cudaError_t output_launch(const Dims& d, const CUtensorMap& mx, const CUtensorMap& mb,
                          const CUtensorMap& mc, const CUtensorMap& my, const TcWorkspace& w,
                          const float* D, void* y, cudaStream_t s)
{
    auto k = block_output_kernel;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, OutSmem::kBytes);
    if (e != cudaSuccess) return e;
    const int hpc = heads_per_cta(d);
    dim3 grid(d.nchunks, d.nheads / hpc, d.batch);
    return launch_dependent(k, grid, dim3(kOutThreads), OutSmem::kBytes, s, mx, mb, mc, my, w.fac,
                            w.himg, D, d.nheads, d.ngroups, d.nchunks, hpc, device_error_word(),
                            static_cast<__nv_bfloat16*>(y), d.cu_seqlens, d.vl_first, d.vl_seq);
}

}  // namespace

bool tc_make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                 CUtensorMapDataType type, uint32_t box_rows)
{
    return make_map(m, base, inner, rows, outer, type, box_rows);
}

int tc_sm_count() { return sm_count(); }

bool tc_encode_map(CUtensorMap* m, CUtensorMapDataType type, int rank, const void* base,
                   const uint64_t* dims, const uint64_t* strides, const uint32_t* box, bool swizzle)
{
    return encode_map(m, type, rank, base, dims, strides, box, swizzle);
}

bool tc_prefill_supported(const Dims& d)
{
    return d.headdim == kP && d.dstate == kN && (d.chunk_len == 128 || d.chunk_len == 256);
}

Dims tc_block_dims(const Dims& d)
{
    Dims t = d;
    t.chunk_len = kBlk;
    t.nchunks = (d.seqlen + kBlk - 1) / kBlk;
    return t;
}

size_t tc_workspace_layout(const Dims& d, void* base, TcWorkspace* w)
{
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t BH = (size_t)d.batch * d.nheads;
    const size_t fac_b = up(BH * d.nchunks * 4 * d.chunk_len * sizeof(float));
    const size_t wts_b = up(BH * d.nchunks * (d.chunk_len + 4) * sizeof(float));
    const size_t himg_b = up(BH * d.nchunks * kHImage);
    const size_t b16_b = up((size_t)d.batch * d.seqlen * d.ngroups * kN * 2);
    const size_t gram_b = up((size_t)d.batch * d.ngroups * d.nchunks * kBlk * kBlk * 2);
    // fused path: a hand-off state (two heads) and flag per CTA boundary that can split a pair
    const size_t slots = d.nseq ? 0 : (size_t)std::min<long long>(fused_units(d), kFusedMaxCtas) + 1;
    const size_t hand_b = up(slots * 2 * kP * kN * sizeof(float));
    const size_t flag_b = up(slots * sizeof(int));
    const size_t mid_b = std::max(wts_b + himg_b, gram_b + hand_b + flag_b);
    if (w) {
        char* p = static_cast<char*>(base);
        w->fac = reinterpret_cast<float*>(p);
        w->wts = reinterpret_cast<float*>(p + fac_b);
        w->himg = reinterpret_cast<uint8_t*>(p + fac_b + wts_b);
        w->gram = reinterpret_cast<uint4*>(p + fac_b);
        w->handoff = reinterpret_cast<float*>(p + fac_b + gram_b);
        w->handoff_flag = reinterpret_cast<int*>(p + fac_b + gram_b + hand_b);
        w->b16 = p + fac_b + mid_b;
    }
    return fac_b + mid_b + b16_b;
}

Dims tc_varlen_dims(int nseq, int total_tokens, int nheads, int headdim, int ngroups, int dstate)
{
    Dims t{1, total_tokens, nheads, headdim, ngroups, dstate, kBlk, total_tokens / kBlk + nseq};
    t.nseq = nseq;
    return t;
}

size_t tc_varlen_workspace_layout(const Dims& t, void* base, TcWorkspace* w, int** first, int** seqof)
{
    auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t main = tc_workspace_layout(t, base, w);
    const size_t first_b = up((size_t)(t.nseq + 1) * sizeof(int));
    const size_t seq_b = up((size_t)t.nchunks * sizeof(int));
    if (first) *first = reinterpret_cast<int*>(static_cast<char*>(base) + main);
    if (seqof) *seqof = reinterpret_cast<int*>(static_cast<char*>(base) + main + first_b);
    return main + first_b + seq_b;
}

cudaError_t launch_varlen_table(const Dims& t, cudaStream_t s)
{
    varlen_table_kernel<<<1, kTableThreads, 0, s>>>(t.cu_seqlens, t.nseq, t.seqlen, t.nchunks, t.chunk_len,
                                                    const_cast<int*>(t.vl_first), const_cast<int*>(t.vl_seq),
                                                    device_error_word());
    return cudaGetLastError();
}

cudaError_t launch_chunk_state_scan_tc(const Dims& d, const void* x, const void* B_f16,
                                       const TcWorkspace& w, const float* init_state,
                                       float* final_state, cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    const uint64_t T = d.seqlen, H = d.nheads, G = d.ngroups, Bt = d.batch;
    WalkMaps m;
    // x [b][T][H][P] bf16 seen as (p, t, h, b): one box = 64 rows of 1 or 2 heads
    const uint64_t xdim[4] = {kP, T, H, Bt};
    const uint64_t xstr[3] = {H * kP * 2, kP * 2, T * H * kP * 2};
    const uint32_t xbox1[4] = {64, 64, 1, 1}, xbox2[4] = {64, 64, 2, 1};
    // fp16 B [b][T][G][N] seen as (n mod 64, t, 2 g + n / 64, b)
    const uint64_t bdim[4] = {64, T, 2 * G, Bt};
    const uint64_t bstr[3] = {G * kN * 2, 128, T * G * kN * 2};
    const uint32_t bbox[4] = {64, 64, 2, 1};
    // weights [b h][c][Q + 4] fp32: a box is 68 floats of the CTA's heads (a stage's 64
    // weights, and for the block's last stage the block decay after them)
    const int nh = walk_heads(d);
    const uint64_t wdim[2] = {(uint64_t)d.nchunks * (d.chunk_len + 4), Bt * H};
    const uint64_t wstr[1] = {(uint64_t)d.nchunks * (d.chunk_len + 4) * 4};
    const uint32_t wbox[2] = {kWRow, (uint32_t)nh};
    if (!encode_map(&m.x1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, x, xdim, xstr, xbox1, true) ||
        !encode_map(&m.x2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, x, xdim, xstr, xbox2, true) ||
        !encode_map(&m.b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, B_f16, bdim, bstr, bbox, true) ||
        !encode_map(&m.w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, w.wts, wdim, wstr, wbox, false))
        return cudaErrorInvalidValue;
    if (d.chunk_len != kBlk) return cudaErrorInvalidValue;
    if (nh == 1) return walk_t<kBlk, 1>(d, m, w, init_state, final_state, s);
    return walk_t<kBlk, 3>(d, m, w, init_state, final_state, s);
}

cudaError_t launch_chunk_output_tc(const Dims& d, const void* x, const void* B, const void* C,
                                   const float* D, const TcWorkspace& w, void* y, cudaStream_t s)
{
    if (d.nchunks == 0 || d.batch == 0) return cudaSuccess;
    CUtensorMap mx, mb, mc, my;
    if (d.chunk_len != kBlk) return cudaErrorInvalidValue;
    if (!make_map(&mx, x, (uint64_t)d.nheads * kP, d.seqlen, d.batch) ||
        !make_map(&mb, B, (uint64_t)d.ngroups * kN, d.seqlen, d.batch) ||
        !make_map(&mc, C, (uint64_t)d.ngroups * kN, d.seqlen, d.batch) ||
        !make_map(&my, y, (uint64_t)d.nheads * kP, d.seqlen, d.batch))
        return cudaErrorInvalidValue;
    return output_launch(d, mx, mb, mc, my, w, D, y, s);
}

}  // namespace ssd
