// Tensor-core (tcgen05 / TMEM / TMA) stages of the bf16 chunked prefill.
#pragma once

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
};
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

}  // namespace ssd
