// Tensor-core (tcgen05 / TMEM / TMA) stages of the bf16 chunked prefill.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace ssd {

// headdim 64, dstate 128, chunk_len 128 or 256, bf16 storage.
bool tc_prefill_supported(const Dims& d);

// The tensor-core stages work in 128-token blocks: the problem with chunk_len = 128 and
// nchunks = ceil(seqlen / 128).  A 256-token chunk is two such blocks, its off-diagonal
// 128 x 128 block entering through the state at its midpoint (an exact factorisation).
Dims tc_block_dims(const Dims& d);

// Workspace of the tensor-core path (sized and indexed by the 128-token block dims).
struct TcWorkspace {
    float* fac;       // [b][h][c][4][Q] Lam (inclusive cumsum of dt A within each block),
                      //   dt (zero past seqlen), and the two column factors of each
                      //   32-token sub-block: exp(Lam_last - Lam_s) dt_s, exp(Lam_first - Lam_s) dt_s
    float* wts;       // [b][h][c][Q + 4] chunk-state weights exp(Lam_end - Lam) dt, then
                      //   exp(Lam_end) and three zeros
    uint8_t* himg;    // [b][h][c] 16 KB bf16 image of each block's start state (MN-major,
                      //   64-byte swizzle: two 8 KB p-halves of [128 n][32 p])
    void* b16;        // [b][T][G][N] fp16 copy of B (operand of the chunk-state GEMM)
    uint4* gram;      // fused path, over wts / himg: [b][g][c] bf16 G = C B^T of each block,
                      //   four planes of 32 columns ([plane][row t][32 bf16])
    float* handoff;   // fused path, after gram: [slot][2 heads][P][N] fp32 states handed from one
                      //   CTA to the next where a head pair's blocks are split between them
    int* handoff_flag;  // fused path: [slot] arrival counts of those hand-offs
};
// Sized for either path: fac, then wts + himg (two-pass) or gram (fused), whichever is
// larger, then b16 (both).
size_t tc_workspace_layout(const Dims& d, void* base, TcWorkspace* w);

// Packed variable-length prefill: the block dims (batch 1, an upper bound of blocks), the
// workspace (the tensor-core workspace, then the block table), and the table kernel.
Dims tc_varlen_dims(int nseq, int total_tokens, int nheads, int headdim, int ngroups, int dstate);
size_t tc_varlen_workspace_layout(const Dims& t, void* base, TcWorkspace* w, int** first, int** seqof);
cudaError_t launch_varlen_table(const Dims& t, cudaStream_t s);

// Chunk states and the inter-chunk recurrence (persistent walk over each head's chunks),
// writing the chunk start states (bf16 images) and the final state.  B_f16 is the fp16
// copy of B.
cudaError_t launch_chunk_state_scan_tc(const Dims& d, const void* x, const void* B_f16,
                                       const TcWorkspace& w, const float* init_state,
                                       float* final_state, cudaStream_t s);

// Per 128-token block: y = (C B^T o L o dt) X + diag(exp Lam) C H_k^T + D x, bf16 out.
cudaError_t launch_chunk_output_tc(const Dims& d, const void* x, const void* B, const void* C,
                                   const float* D, const TcWorkspace& w, void* y, cudaStream_t s);

// Fused path (batched, not packed variable-length), launched after the cumsum kernel:
// G = C B^T of every block (bf16, w.gram; the same launch clears the hand-off flags); then
// one kernel whose CTAs walk the blocks of head pairs with the pairs' states in TMEM and
// write y and the final state.  Both are programmatic dependents; the G kernel completes
// only after the cumsum kernel has.
cudaError_t launch_block_gram(const Dims& d, const void* B, const void* C, const TcWorkspace& w,
                              cudaStream_t s);
// The chain kernel reads the fp16 copy of B (w.b16) that the cumsum kernel writes.
cudaError_t launch_chain_prefill(const Dims& d, const void* x, const void* C, const float* D,
                                 const TcWorkspace& w, const float* init_state, float* final_state,
                                 void* y, cudaStream_t s);

// Fused path: the head pairs' chains and the hand-off slots they may need (one per CTA
// boundary, at most kFusedMaxCtas + 1).
constexpr int kFusedMaxCtas = 256;
bool fused_prefill_supported(const Dims& d);
long long fused_units(const Dims& d);

// helpers shared by the tensor-core launchers
// 16-bit tensor [outer][rows][inner] read in boxes of 64 (inner) x box_rows, 128-byte swizzle.
bool tc_make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                 CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint32_t box_rows = 128);
// Tiled map of `rank` dimensions (dim 0 contiguous, strides in bytes for dims 1..rank-1),
// 128-byte swizzle or none.
bool tc_encode_map(CUtensorMap* m, CUtensorMapDataType type, int rank, const void* base,
                   const uint64_t* dims, const uint64_t* strides, const uint32_t* box, bool swizzle);
int tc_sm_count();

// Launch with programmatic stream serialisation: the kernel may start while the previous
// kernel of the stream finishes, and waits (griddepcontrol.wait) before reading its output.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace ssd
