// Self-test of the library's bounded device waits.  One CTA waits on an mbarrier that
// nothing arrives on and on a global flag that nothing sets, each with a short
// iteration limit, using the same wait helpers as the prefill kernels.  Both waits
// expire, record SSD_ERR_TIMEOUT in the device error word and return; nothing traps and
// nothing hangs, so the context stays usable.
#include "ptx.cuh"

namespace ssd {
namespace {

__global__ void bounded_wait_selftest_kernel(const int* flag, int* err, uint32_t max_iters,
                                             int* outcome)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool mbar_done = ptx::mbar_wait(&bar, 0, err, max_iters);
        const bool flag_done = ptx::wait_flag_geq(flag, 1, err, max_iters);
        outcome[0] = mbar_done ? 1 : 0;
        outcome[1] = flag_done ? 1 : 0;
        // complete the barrier phase so that no wait is left pending at exit
        ptx::mbar_arrive(&bar);
    }
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status_t ssd_selftest_bounded_waits(int* scratch, void* stream)
{
    if (!scratch) return SSD_ERR_NULL;
    int* err = ssd::device_error_word();
    if (!err) return SSD_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(scratch, 0, 3 * sizeof(int), s) != cudaSuccess) return SSD_ERR_CUDA;
    // scratch[0]: the flag nothing sets; scratch[1..2]: whether each wait completed
    ssd::bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(scratch, err, 1u << 16, scratch + 1);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
