// Tensor-core (tcgen05 / TMEM / TMA) stages of the bf16 chunked prefill.
#pragma once

#include "common.cuh"

namespace ssd {

// headdim 64, dstate 128, chunk_len 128 or 256, bf16 storage.
bool tc_prefill_supported(const Dims& d);

// Chunk states S_c = B_c^T (w o X_c), w_s = exp(Lam_end - Lam_s) dt_s, written
// fp32 [b][h][c][headdim][dstate].
cudaError_t launch_chunk_state_tc(const Dims& d, const void* x, const float* dt, const void* B,
                                  const float* lam, float* states, cudaStream_t s);

// y = (C B^T o L o dt) X + diag(exp Lam) C H_c^T + D x, bf16 out.
cudaError_t launch_chunk_output_tc(const Dims& d, const void* x, const float* dt, const void* B,
                                   const void* C, const float* D, const float* lam,
                                   const float* states, void* y, cudaStream_t s);

}  // namespace ssd
