// ssd_prefill_noalloc: the chunked prefill for callers that cannot allocate device
// memory.
//
// Some callers are not allowed to allocate: code that runs inside a host framework's
// execution hook (an inference runtime's plugin enqueue, for example) must work in
// the memory the framework planned, and code that runs while a stream is being
// captured into a CUDA graph cannot call cudaMalloc without breaking the capture.
// ssd_prefill needs a caller-provided workspace (per-chunk decay sums and per-chunk
// states); this entry point supplies it from a fixed buffer that lives in the
// library's own device image instead, so the caller passes only inputs and outputs.
//
// The buffer is a file-scope __device__ array of kNoAllocScratchBytes (64 MiB).  Every
// GPU that loads this library holds it until the process exits.  Problems whose
// workspace would exceed it are rejected with SSD_ERR_WORKSPACE before anything is
// launched.  All calls share the one buffer, so calls that overlap on the GPU (for
// example on two streams) race on it and must be serialised by the caller.  Nothing
// in the buffer has to start at zero: every byte a call reads was written earlier by
// the same call, and the previous call's contents are simply overwritten.
//
// In host code the array's name is only a host-side stand-in for the symbol, not a
// device address; its device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) on the first call made while that
// device is current.  That first call should therefore happen before any stream
// capture that includes this entry point.  The lookup is serialised by a mutex, so two
// host threads making their first call at once both get the one address.  The cached
// address belongs to the device's primary context (the one the CUDA runtime uses): a
// caller that resets the device (cudaDeviceReset) must not call this entry point again
// in the same process, since the cached address would then be stale.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device (nullptr on failure).
void* scratch_on_current_device()
{
    static std::mutex lock;
    static void* addr[kMaxDevices] = {nullptr};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> hold(lock);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" ssd_status_t ssd_prefill_noalloc(const void* x, const float* dt, const float* A,
                                            const void* B, const void* C, const float* D,
                                            const float* init_state, int batch, int seqlen,
                                            int nheads, int headdim, int ngroups, int dstate,
                                            int chunk_len, ssd_dtype_t dtype, void* y,
                                            float* final_state, void* stream)
{
    const size_t need = ssd_prefill_workspace_bytes(batch, seqlen, nheads, headdim, ngroups,
                                                    dstate, chunk_len, dtype);
    if (need > kNoAllocScratchBytes) return SSD_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = scratch_on_current_device();
        if (!scratch) return SSD_ERR_CUDA;
    }
    return ssd_prefill(x, dt, A, B, C, D, init_state, batch, seqlen, nheads, headdim, ngroups,
                       dstate, chunk_len, dtype, y, final_state, scratch,
                       need > 0 ? kNoAllocScratchBytes : 0, stream);
}
