// Device-side seeded input generator (random draws only; see include/ssd_inputs.h).
// Philox4x32-10 as published by Salmon et al. (SC'11); Irwin-Hall normals formed in
// integers so that the host twin reproduces every value exactly.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd_inputs.h"

namespace {

constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;

__device__ __forceinline__ uint4 philox10(uint4 c, uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t lo0 = kM0 * c.x, hi0 = __umulhi(kM0, c.x);
        const uint32_t lo1 = kM1 * c.z, hi1 = __umulhi(kM1, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += kW0;
        k1 += kW1;
    }
    return c;
}

__global__ void gen_normal_kernel(float* out, size_t n, uint32_t k0, uint32_t k1, uint32_t sid,
                                  float scale, uint64_t first)
{
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        const uint64_t idx = first + i;
        int32_t total = 0;
#pragma unroll
        for (uint32_t j = 0; j < 3; ++j) {
            const uint4 w = philox10(make_uint4((uint32_t)idx, sid, j, (uint32_t)(idx >> 32)), k0, k1);
            total += (int32_t)(w.x >> 8) + (int32_t)(w.y >> 8) + (int32_t)(w.z >> 8) + (int32_t)(w.w >> 8);
        }
        const int32_t centred = total - 6 * (1 << 24);
        const float z = __int2float_rn(centred) * 0x1p-24f;   // exact power-of-two scaling
        out[i] = __fmul_rn(z, scale);
    }
}

__global__ void gen_table_kernel(float* out, size_t n, const float* table, int bits, uint32_t k0,
                                 uint32_t k1, uint32_t sid, uint64_t first)
{
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        const uint64_t idx = first + i;
        const uint4 w = philox10(make_uint4((uint32_t)idx, sid, 3u, (uint32_t)(idx >> 32)), k0, k1);
        out[i] = table[w.x >> (32 - bits)];
    }
}

unsigned grid_for(size_t n)
{
    const size_t blocks = (n + 255) / 256;
    return (unsigned)(blocks < 148 * 64 ? (blocks ? blocks : 1) : 148 * 64);
}

}  // namespace

extern "C" int ssd_gen_normal(float* out, size_t n, uint64_t seed, uint32_t philox_stream,
                              float scale, uint64_t first_index, void* stream)
{
    if (n == 0) return 0;
    if (!out) return (int)cudaErrorInvalidValue;
    gen_normal_kernel<<<grid_for(n), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        out, n, (uint32_t)seed, (uint32_t)(seed >> 32), philox_stream, scale, first_index);
    return (int)cudaGetLastError();
}

extern "C" int ssd_gen_table(float* out, size_t n, const float* table, int bits, uint64_t seed,
                             uint32_t philox_stream, uint64_t first_index, void* stream)
{
    if (n == 0) return 0;
    if (!out || !table || bits < 1 || bits > 24) return (int)cudaErrorInvalidValue;
    gen_table_kernel<<<grid_for(n), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        out, n, table, bits, (uint32_t)seed, (uint32_t)(seed >> 32), philox_stream, first_index);
    return (int)cudaGetLastError();
}
