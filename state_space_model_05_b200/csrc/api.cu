// C ABI of the SSD library: argument validation, workspace sizing and dispatch.
// Every entry point validates on the host before launching anything and only
// enqueues work on the caller's stream.
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <vector>

#include "common.cuh"
#include "prefill_tc.h"

namespace ssd {

__device__ int g_error_word = 0;

int* device_error_word()
{
    static int* cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<int*>(p);
    }
    return cache[dev];
}

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ssd_status_t check_common(int batch, int nheads, int headdim, int ngroups, int dstate,
                          ssd_dtype_t dtype, int max_dstate)
{
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_DTYPE;
    if (batch < 0 || batch > 65535) return SSD_ERR_SHAPE;
    if (nheads < 1 || nheads > 65535 || ngroups < 1 || nheads % ngroups != 0) return SSD_ERR_SHAPE;
    if (headdim < 8 || headdim % 8 != 0 || dstate < 8 || dstate % 8 != 0) return SSD_ERR_SHAPE;
    if (headdim > 128 || dstate > max_dstate) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

ssd_status_t prefill_dims(int batch, int seqlen, int nheads, int headdim, int ngroups, int dstate,
                          int chunk_len, ssd_dtype_t dtype, Dims* d)
{
    ssd_status_t st = check_common(batch, nheads, headdim, ngroups, dstate, dtype, 256);
    if (st != SSD_OK) return st;
    if (seqlen < 0 || chunk_len < 1) return SSD_ERR_SHAPE;
    if (chunk_len > 256) return SSD_ERR_UNSUPPORTED;
    d->batch = batch;
    d->seqlen = seqlen;
    d->nheads = nheads;
    d->headdim = headdim;
    d->ngroups = ngroups;
    d->dstate = dstate;
    d->chunk_len = chunk_len;
    d->nchunks = (seqlen + chunk_len - 1) / chunk_len;
    return SSD_OK;
}

ssd_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA; }

// ---- opt-in kernel profiling: an event pair around each launch -------------------
enum Stage { kCumsum, kStateTc, kStateSimt, kScan, kOutTc, kOutSimt, kDecode, kCopy, kDecodeLayers, kGdn,
             kGram, kChain, kDecodeSteps, kDecodeStepsLayers, kNumStages };
const char* const kStageNames[kNumStages] = {"chunk_cumsum", "chunk_state_scan_tc", "chunk_state_simt",
                                              "state_scan", "chunk_output_tc", "chunk_output_simt",
                                              "decode_step", "copy_state", "decode_step_layers",
                                              "gdn_decode_step", "block_gram_tc", "chain_prefill_tc",
                                              "decode_steps", "decode_steps_layers"};

// which tensor-core prefill batched calls take (ssd_set_prefill_path)
std::atomic<int> g_prefill_path{SSD_PREFILL_AUTO};
struct ProfRecord { int stage; cudaEvent_t begin, end; };
struct Profiler {
    bool on = false;
    std::vector<ProfRecord> records;
    std::vector<cudaEvent_t> pool;
    size_t used = 0;
    cudaEvent_t next() {
        if (used == pool.size()) {
            cudaEvent_t e = nullptr;
            if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
            pool.push_back(e);
        }
        return pool[used++];
    }
};
Profiler g_prof;

// Runs `launch` between two profiling events when profiling is enabled.
template <typename F>
cudaError_t profiled(int stage, cudaStream_t s, F&& launch)
{
    if (!g_prof.on) return launch();
    cudaEvent_t a = g_prof.next(), b = g_prof.next();
    // inside a stream capture an event record must be marked external to become a
    // timed record node of the graph (otherwise it is only a dependency marker)
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cap);
    const unsigned flags = cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : 0u;
    if (a) cudaEventRecordWithFlags(a, s, flags);
    const cudaError_t e = launch();
    if (b) cudaEventRecordWithFlags(b, s, flags);
    if (a && b) g_prof.records.push_back({stage, a, b});
    return e;
}

}  // namespace

size_t prefill_workspace_layout(const Dims& d, void* base, PrefillWorkspace* ws)
{
    const size_t units = (size_t)d.batch * d.nheads * d.nchunks;
    const size_t lam_bytes = align_up(units * 2 * d.chunk_len * sizeof(float));   // hi and lo parts
    const size_t st_bytes = align_up(units * d.headdim * d.dstate * sizeof(float));
    if (ws) {
        char* p = static_cast<char*>(base);
        ws->lam = reinterpret_cast<float*>(p);
        ws->states = reinterpret_cast<float*>(p + lam_bytes);
    }
    return lam_bytes + st_bytes;
}

}  // namespace ssd

using namespace ssd;

extern "C" {

int ssd_abi_version(void) { return 101; }

const char* ssd_status_string(ssd_status_t s)
{
    switch (s) {
        case SSD_OK: return "ok";
        case SSD_ERR_NULL: return "a required pointer is NULL";
        case SSD_ERR_SHAPE: return "invalid or inconsistent sizes";
        case SSD_ERR_DTYPE: return "unknown dtype";
        case SSD_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case SSD_ERR_UNSUPPORTED: return "shape not supported by this build";
        case SSD_ERR_CUDA: return "CUDA error";
        case SSD_ERR_TIMEOUT: return "device-side bounded wait expired";
        case SSD_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

size_t ssd_prefill_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int ngroups,
                                   int dstate, int chunk_len, ssd_dtype_t dtype)
{
    Dims d;
    if (prefill_dims(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_len, dtype, &d) != SSD_OK)
        return 0;
    if (d.nchunks == 0 || d.batch == 0) return 0;
    if (dtype == SSD_BF16 && tc_prefill_supported(d))
        return tc_workspace_layout(tc_block_dims(d), nullptr, nullptr);
    return prefill_workspace_layout(d, nullptr, nullptr);
}

namespace {

// ssd_prefill and ssd_prefill_dtraw: dt_softplus selects dt = softplus(dt_in + dt_bias[h]).
ssd_status_t prefill_impl(const void* x, const float* dt, const float* dt_bias, int dt_softplus,
                          const float* A, const void* B, const void* C, const float* D,
                          const float* init_state, int batch, int seqlen, int nheads, int headdim,
                          int ngroups, int dstate, int chunk_len, ssd_dtype_t dtype, void* y,
                          float* final_state, void* workspace, size_t workspace_bytes, void* stream)
{
    Dims d;
    ssd_status_t st = prefill_dims(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_len,
                                   dtype, &d);
    if (st != SSD_OK) return st;
    if (dt_softplus && dt_bias && !aligned16(dt_bias)) return SSD_ERR_ALIGN;
    d.dt_bias = dt_bias;
    d.dt_softplus = dt_softplus;
    if (batch == 0) return SSD_OK;
    if (!final_state) return SSD_ERR_NULL;
    if (!aligned16(final_state) || !aligned16(init_state)) return SSD_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (seqlen == 0)
        return from_cuda(profiled(kCopy, s, [&] { return launch_copy_state(d, init_state, final_state, s); }));

    if (!x || !dt || !A || !B || !C || !D || !y) return SSD_ERR_NULL;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(A) || !aligned16(B) || !aligned16(C) ||
        !aligned16(D) || !aligned16(y) || !aligned16(workspace))
        return SSD_ERR_ALIGN;
    const bool tc = dtype == SSD_BF16 && tc_prefill_supported(d);
    if (tc) {
        const Dims t = tc_block_dims(d);
        TcWorkspace w;
        const size_t need = tc_workspace_layout(t, workspace, &w);
        if (!workspace || workspace_bytes < need) return SSD_ERR_WORKSPACE;
        if (g_prefill_path.load() == SSD_PREFILL_FUSED && fused_prefill_supported(t)) {
            // fused: decay factors, G = C B^T per block, then the chain kernel
            cudaError_t e = profiled(kCumsum, s, [&] {
                return launch_chunk_cumsum(t, dt, A, w.fac, true, nullptr, B, w.b16, s);
            });
            if (e == cudaSuccess) e = profiled(kGram, s, [&] { return launch_block_gram(t, B, C, w, s); });
            if (e == cudaSuccess)
                e = profiled(kChain, s, [&] {
                    return launch_chain_prefill(t, x, C, D, w, init_state, final_state, y, s);
                });
            return from_cuda(e);
        }
        cudaError_t e = profiled(kCumsum, s, [&] {
            return launch_chunk_cumsum(t, dt, A, w.fac, true, w.wts, B, w.b16, s);
        });
        if (e == cudaSuccess)
            e = profiled(kStateTc, s, [&] {
                return launch_chunk_state_scan_tc(t, x, w.b16, w, init_state, final_state, s);
            });
        if (e == cudaSuccess)
            e = profiled(kOutTc, s, [&] { return launch_chunk_output_tc(t, x, B, C, D, w, y, s); });
        return from_cuda(e);
    }

    PrefillWorkspace ws;
    const size_t need = prefill_workspace_layout(d, workspace, &ws);
    if (!workspace || workspace_bytes < need) return SSD_ERR_WORKSPACE;
    cudaError_t e = profiled(kCumsum, s, [&] {
        return launch_chunk_cumsum(d, dt, A, ws.lam, false, nullptr, nullptr, nullptr, s);
    });
    if (e == cudaSuccess)
        e = profiled(kStateSimt, s, [&] {
            return launch_chunk_state_simt(d, dtype, x, dt, B, ws.lam, ws.states, s);
        });
    if (e == cudaSuccess)
        e = profiled(kScan, s, [&] {
            return launch_state_scan(d, ws.lam, ws.states, init_state, final_state, s);
        });
    if (e == cudaSuccess)
        e = profiled(kOutSimt, s, [&] {
            return launch_chunk_output_simt(d, dtype, x, dt, B, C, D, ws.lam, ws.states, y, s);
        });
    return from_cuda(e);
}

}  // namespace

namespace {

ssd_status_t varlen_dims(int nseq, int total_tokens, int nheads, int headdim, int ngroups, int dstate,
                         int chunk_len, ssd_dtype_t dtype, Dims* t, bool* tc)
{
    ssd_status_t st = check_common(1, nheads, headdim, ngroups, dstate, dtype, 256);
    if (st != SSD_OK) return st;
    if (nseq < 1 || nseq > (1 << 20) || total_tokens < 0 || chunk_len < 1) return SSD_ERR_SHAPE;
    if (chunk_len > 256) return SSD_ERR_UNSUPPORTED;
    Dims d{1, total_tokens, nheads, headdim, ngroups, dstate, chunk_len, 1};
    *tc = dtype == SSD_BF16 && tc_prefill_supported(d);
    if (*tc) {
        *t = tc_varlen_dims(nseq, total_tokens, nheads, headdim, ngroups, dstate);
    } else {
        // CUDA-core path: chunks of chunk_len, at most floor(T / Q) + nseq of them
        *t = Dims{1, total_tokens, nheads, headdim, ngroups, dstate, chunk_len, total_tokens / chunk_len + nseq};
        t->nseq = nseq;
    }
    return SSD_OK;
}

// the CUDA-core workspace, then the block table (first [nseq + 1], sequence of each chunk)
size_t simt_varlen_workspace_layout(const Dims& t, void* base, PrefillWorkspace* ws, int** first, int** seqof)
{
    const size_t main = prefill_workspace_layout(t, base, ws);
    const size_t first_b = align_up((size_t)(t.nseq + 1) * sizeof(int));
    const size_t seq_b = align_up((size_t)t.nchunks * sizeof(int));
    if (first) *first = reinterpret_cast<int*>(static_cast<char*>(base) + main);
    if (seqof) *seqof = reinterpret_cast<int*>(static_cast<char*>(base) + main + first_b);
    return main + first_b + seq_b;
}

}  // namespace

size_t ssd_prefill_varlen_workspace_bytes(int nseq, int total_tokens, int nheads, int headdim,
                                          int ngroups, int dstate, int chunk_len, ssd_dtype_t dtype)
{
    Dims t;
    bool tc = false;
    if (varlen_dims(nseq, total_tokens, nheads, headdim, ngroups, dstate, chunk_len, dtype, &t, &tc) != SSD_OK)
        return 0;
    if (total_tokens == 0) return 0;
    return tc ? tc_varlen_workspace_layout(t, nullptr, nullptr, nullptr, nullptr)
              : simt_varlen_workspace_layout(t, nullptr, nullptr, nullptr, nullptr);
}

ssd_status_t ssd_prefill_varlen(const void* x, const float* dt, const float* A, const void* B,
                                const void* C, const float* D, const float* init_states,
                                const int* cu_seqlens, int nseq, int total_tokens, int nheads,
                                int headdim, int ngroups, int dstate, int chunk_len, ssd_dtype_t dtype,
                                void* y, float* final_states, void* workspace, size_t workspace_bytes,
                                void* stream)
{
    Dims t;
    bool tc = false;
    ssd_status_t st = varlen_dims(nseq, total_tokens, nheads, headdim, ngroups, dstate, chunk_len, dtype, &t, &tc);
    if (st != SSD_OK) return st;
    if (!final_states || !cu_seqlens) return SSD_ERR_NULL;
    if (!aligned16(final_states) || !aligned16(init_states) || reinterpret_cast<uintptr_t>(cu_seqlens) % 4)
        return SSD_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (total_tokens == 0) {
        Dims c{nseq, 0, nheads, headdim, ngroups, dstate, chunk_len, 0};
        return from_cuda(profiled(kCopy, s, [&] { return launch_copy_state(c, init_states, final_states, s); }));
    }
    if (!x || !dt || !A || !B || !C || !D || !y) return SSD_ERR_NULL;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(A) || !aligned16(B) || !aligned16(C) ||
        !aligned16(D) || !aligned16(y) || !aligned16(workspace))
        return SSD_ERR_ALIGN;
    int* first = nullptr;
    int* seqof = nullptr;
    t.cu_seqlens = cu_seqlens;
    if (tc) {
        TcWorkspace w;
        const size_t need = tc_varlen_workspace_layout(t, workspace, &w, &first, &seqof);
        if (!workspace || workspace_bytes < need) return SSD_ERR_WORKSPACE;
        t.vl_first = first;
        t.vl_seq = seqof;
        cudaError_t e = profiled(kCumsum, s, [&] {
            cudaError_t r = launch_varlen_table(t, s);
            return r != cudaSuccess ? r : launch_chunk_cumsum(t, dt, A, w.fac, true, w.wts, B, w.b16, s);
        });
        if (e == cudaSuccess)
            e = profiled(kStateTc, s, [&] {
                return launch_chunk_state_scan_tc(t, x, w.b16, w, init_states, final_states, s);
            });
        if (e == cudaSuccess)
            e = profiled(kOutTc, s, [&] { return launch_chunk_output_tc(t, x, B, C, D, w, y, s); });
        return from_cuda(e);
    }
    PrefillWorkspace ws;
    const size_t need = simt_varlen_workspace_layout(t, workspace, &ws, &first, &seqof);
    if (!workspace || workspace_bytes < need) return SSD_ERR_WORKSPACE;
    t.vl_first = first;
    t.vl_seq = seqof;
    cudaError_t e = profiled(kCumsum, s, [&] {
        cudaError_t r = launch_varlen_table(t, s);
        return r != cudaSuccess ? r : launch_chunk_cumsum(t, dt, A, ws.lam, false, nullptr, nullptr, nullptr, s);
    });
    if (e == cudaSuccess)
        e = profiled(kStateSimt, s, [&] { return launch_chunk_state_simt(t, dtype, x, dt, B, ws.lam, ws.states, s); });
    if (e == cudaSuccess)
        e = profiled(kScan, s, [&] { return launch_state_scan(t, ws.lam, ws.states, init_states, final_states, s); });
    if (e == cudaSuccess)
        e = profiled(kOutSimt, s, [&] {
            return launch_chunk_output_simt(t, dtype, x, dt, B, C, D, ws.lam, ws.states, y, s);
        });
    return from_cuda(e);
}

ssd_status_t ssd_prefill(const void* x, const float* dt, const float* A, const void* B,
                         const void* C, const float* D, const float* init_state, int batch,
                         int seqlen, int nheads, int headdim, int ngroups, int dstate,
                         int chunk_len, ssd_dtype_t dtype, void* y, float* final_state,
                         void* workspace, size_t workspace_bytes, void* stream)
{
    return prefill_impl(x, dt, nullptr, 0, A, B, C, D, init_state, batch, seqlen, nheads, headdim,
                        ngroups, dstate, chunk_len, dtype, y, final_state, workspace, workspace_bytes,
                        stream);
}

ssd_status_t ssd_set_prefill_path(ssd_prefill_path_t path)
{
    if (path != SSD_PREFILL_AUTO && path != SSD_PREFILL_FUSED && path != SSD_PREFILL_TWO_PASS)
        return SSD_ERR_SHAPE;
    g_prefill_path.store(path);
    return SSD_OK;
}

ssd_prefill_path_t ssd_get_prefill_path(void) { return static_cast<ssd_prefill_path_t>(g_prefill_path.load()); }

ssd_status_t ssd_prefill_dtraw(const void* x, const float* dt_raw, const float* dt_bias,
                               const float* A, const void* B, const void* C, const float* D,
                               const float* init_state, int batch, int seqlen, int nheads,
                               int headdim, int ngroups, int dstate, int chunk_len,
                               ssd_dtype_t dtype, void* y, float* final_state, void* workspace,
                               size_t workspace_bytes, void* stream)
{
    return prefill_impl(x, dt_raw, dt_bias, 1, A, B, C, D, init_state, batch, seqlen, nheads, headdim,
                        ngroups, dstate, chunk_len, dtype, y, final_state, workspace, workspace_bytes,
                        stream);
}

ssd_status_t ssd_gdn_decode_step(float* state, const void* q, const void* k, const void* v,
                                 const float* gate, const float* beta, int batch, int heads_qk,
                                 int heads_v, int dk, int dv, ssd_dtype_t dtype, void* out,
                                 void* stream)
{
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_DTYPE;
    if (batch < 0 || heads_qk <= 0 || heads_v <= 0 || heads_v % heads_qk != 0 || dk <= 0 || dv <= 0 ||
        dk % 8 != 0 || dv % 4 != 0)
        return SSD_ERR_SHAPE;
    if (!gdn_sizes_supported(dk, dv)) return SSD_ERR_UNSUPPORTED;
    if ((long long)batch * heads_v > 0x7fffffffLL) return SSD_ERR_SHAPE;
    if (batch == 0) return SSD_OK;
    if (!state || !q || !k || !v || !gate || !beta || !out) return SSD_ERR_NULL;
    if (!aligned16(state) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) ||
        !aligned16(beta) || !aligned16(out))
        return SSD_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return from_cuda(profiled(kGdn, s, [&] {
        return launch_gdn_decode(dtype, state, q, k, v, gate, beta, out, batch, heads_qk, heads_v, dk, dv, s);
    }));
}

ssd_status_t ssd_decode_step_layers(const ssd_decode_layer_t* layers, int n_layers, int batch,
                                    int nheads, int headdim, int ngroups, int dstate,
                                    ssd_dtype_t dtype, void* stream)
{
    ssd_status_t st = check_common(batch, nheads, headdim, ngroups, dstate, dtype, 512);
    if (st != SSD_OK) return st;
    if (n_layers < 0 || n_layers > 65535) return SSD_ERR_SHAPE;
    if (batch == 0 || n_layers == 0) return SSD_OK;
    if (!layers) return SSD_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(layers) % alignof(ssd_decode_layer_t)) return SSD_ERR_ALIGN;
    Dims d{batch, 1, nheads, headdim, ngroups, dstate, 1, 1};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return from_cuda(profiled(kDecodeLayers, s, [&] {
        return launch_decode_layers(d, dtype, layers, n_layers, s);
    }));
}

ssd_status_t ssd_decode_steps_layers(const ssd_decode_layer_t* layers, int n_layers, int steps, int batch,
                                     int nheads, int headdim, int ngroups, int dstate, ssd_dtype_t dtype,
                                     void* stream)
{
    ssd_status_t st = check_common(batch, nheads, headdim, ngroups, dstate, dtype, 512);
    if (st != SSD_OK) return st;
    if (n_layers < 0 || n_layers > 65535 || steps < 0) return SSD_ERR_SHAPE;
    if (batch == 0 || n_layers == 0 || steps == 0) return SSD_OK;
    if (!layers) return SSD_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(layers) % alignof(ssd_decode_layer_t)) return SSD_ERR_ALIGN;
    Dims d{batch, 1, nheads, headdim, ngroups, dstate, 1, 1};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return from_cuda(profiled(kDecodeStepsLayers, s, [&] {
        return launch_decode_steps_layers(d, dtype, layers, n_layers, steps, s);
    }));
}

namespace {

ssd_status_t decode_impl(float* state, const void* x_t, const float* dt_t, const float* dt_bias,
                         int dt_softplus, const float* A, const void* B_t, const void* C_t,
                         const float* D, int batch, int nheads, int headdim, int ngroups, int dstate,
                         ssd_dtype_t dtype, void* y_t, void* stream)
{
    ssd_status_t st = check_common(batch, nheads, headdim, ngroups, dstate, dtype, 512);
    if (st != SSD_OK) return st;
    if (batch == 0) return SSD_OK;
    if (!state || !x_t || !dt_t || !A || !B_t || !C_t || !D || !y_t) return SSD_ERR_NULL;
    if (!aligned16(state) || !aligned16(x_t) || !aligned16(dt_t) || !aligned16(A) ||
        !aligned16(B_t) || !aligned16(C_t) || !aligned16(D) || !aligned16(y_t) ||
        (dt_softplus && dt_bias && !aligned16(dt_bias)))
        return SSD_ERR_ALIGN;
    Dims d{batch, 1, nheads, headdim, ngroups, dstate, 1, 1};
    d.dt_bias = dt_bias;
    d.dt_softplus = dt_softplus;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return from_cuda(profiled(kDecode, s, [&] {
        return launch_decode(d, dtype, state, x_t, dt_t, A, B_t, C_t, D, y_t, s);
    }));
}

}  // namespace

ssd_status_t ssd_decode_step(float* state, const void* x_t, const float* dt_t, const float* A,
                             const void* B_t, const void* C_t, const float* D, int batch,
                             int nheads, int headdim, int ngroups, int dstate, ssd_dtype_t dtype,
                             void* y_t, void* stream)
{
    return decode_impl(state, x_t, dt_t, nullptr, 0, A, B_t, C_t, D, batch, nheads, headdim, ngroups,
                       dstate, dtype, y_t, stream);
}

ssd_status_t ssd_decode_steps(float* state, const void* x, const float* dt, const float* A, const void* B,
                              const void* C, const float* D, int steps, int batch, int nheads, int headdim,
                              int ngroups, int dstate, ssd_dtype_t dtype, void* y, void* stream)
{
    ssd_status_t st = check_common(batch, nheads, headdim, ngroups, dstate, dtype, 512);
    if (st != SSD_OK) return st;
    if (steps < 0) return SSD_ERR_SHAPE;
    if (batch == 0 || steps == 0) return SSD_OK;
    if (!state || !x || !dt || !A || !B || !C || !D || !y) return SSD_ERR_NULL;
    if (!aligned16(state) || !aligned16(x) || !aligned16(dt) || !aligned16(A) || !aligned16(B) ||
        !aligned16(C) || !aligned16(D) || !aligned16(y))
        return SSD_ERR_ALIGN;
    Dims d{batch, 1, nheads, headdim, ngroups, dstate, 1, 1};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return from_cuda(profiled(kDecodeSteps, s, [&] {
        return launch_decode_steps(d, dtype, steps, state, x, dt, A, B, C, D, y, s);
    }));
}

ssd_status_t ssd_decode_step_dtraw(float* state, const void* x_t, const float* dt_raw_t,
                                   const float* dt_bias, const float* A, const void* B_t,
                                   const void* C_t, const float* D, int batch, int nheads,
                                   int headdim, int ngroups, int dstate, ssd_dtype_t dtype,
                                   void* y_t, void* stream)
{
    return decode_impl(state, x_t, dt_raw_t, dt_bias, 1, A, B_t, C_t, D, batch, nheads, headdim, ngroups,
                       dstate, dtype, y_t, stream);
}

ssd_status_t ssd_device_status(void* stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SSD_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int)) != cudaSuccess) return SSD_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return SSD_ERR_CUDA;
        return static_cast<ssd_status_t>(word);
    }
    return SSD_OK;
}

void ssd_profile_enable(int on) { g_prof.on = on != 0; }

void ssd_profile_reset(void)
{
    g_prof.records.clear();
    g_prof.used = 0;
}

int ssd_profile_read(int max_kernels, const char** names, double* total_ms, long long* launches)
{
    double ms[kNumStages] = {0};
    long long n[kNumStages] = {0};
    for (const ProfRecord& r : g_prof.records) {
        if (cudaEventSynchronize(r.end) != cudaSuccess) return -1;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, r.begin, r.end) != cudaSuccess) return -1;
        ms[r.stage] += t;
        n[r.stage] += 1;
    }
    int k = 0;
    for (int i = 0; i < kNumStages && k < max_kernels; ++i) {
        if (n[i] == 0) continue;
        if (names) names[k] = kStageNames[i];
        if (total_ms) total_ms[k] = ms[i];
        if (launches) launches[k] = n[i];
        ++k;
    }
    return k;
}

}  // extern "C"
