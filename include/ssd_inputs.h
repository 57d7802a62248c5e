/*
 * ssd_inputs.h -- device-side seeded input generator for large synthetic SSD workloads.
 *
 * Random draws only (no part of the SSD computation).  It exists for workloads
 * whose inputs are too large to draw on the host (a 64-layer decode stack holds
 * ~43 GB of states and draws fresh per-layer inputs every step).  The host-side
 * twin in state_space_model_05_b200/inputs.py implements the same published
 * definitions independently, so both sides produce bit-identical values:
 *
 *   Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
 *   as 1, 2, 3", SC'11) with key (seed lo, seed hi).  Element i of stream s uses
 *   counters (i lo, s, j, i hi):
 *     normal : j = 0, 1, 2 -> twelve 32-bit words; the top 24 bits of each are
 *              summed in integers (Irwin-Hall), centred by 6 * 2^24, converted to
 *              fp32 once (round to nearest even) and scaled by 2^-24, then
 *              multiplied by `scale` in fp32;
 *     table  : j = 3 -> the top `bits` bits of the first word index `table`.
 *
 * Both calls are asynchronous on `stream` (a cudaStream_t as void*); they return 0,
 * or a nonzero CUDA error code.  `out` is device memory holding n floats; `table`
 * is device memory holding 2^bits floats.
 */
#ifndef SSD_INPUTS_H
#define SSD_INPUTS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int ssd_gen_normal(float* out, size_t n, uint64_t seed, uint32_t philox_stream, float scale,
                   uint64_t first_index, void* stream);

int ssd_gen_table(float* out, size_t n, const float* table, int bits, uint64_t seed,
                  uint32_t philox_stream, uint64_t first_index, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SSD_INPUTS_H */
