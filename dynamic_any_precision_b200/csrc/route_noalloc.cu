// Router entry point that allocates nothing, for callers that cannot call cudaMalloc.
//
// dpa_route needs a caller-provided workspace (per-token counters and a logits buffer).
// Some callers cannot provide one: a plugin running inside a host engine that owns every
// byte of device memory, code that must stay clear of the allocator's implicit device
// synchronisation, or a latency-critical loop that may not allocate at all. This variant
// keeps its scratch in a fixed array in the library's own device memory instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the library holds it
// (kNoAllocScratchBytes) until the process exits. Its host-side name is only a handle: the
// device address is looked up with cudaGetSymbolAddress once per device, with that device
// current, the first time this entry point runs on it (so make that first call before any
// stream capture begins).
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "common.cuh"
#include "dpa.h"
#include "kernels.h"

namespace {

constexpr int kNoAllocMaxTokens = 1024;
constexpr int kNoAllocMaxLogits = 65536;   // n_tokens * n_experts
constexpr size_t kCountersOff = 256;       // after the error header
constexpr size_t kLogitsOff = kCountersOff + sizeof(unsigned) * kNoAllocMaxTokens;
constexpr size_t kNoAllocScratchBytes = kLogitsOff + sizeof(double) * kNoAllocMaxLogits;

static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once per device).
dpa_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DPA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return DPA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return DPA_OK;
}

}  // namespace

extern "C" dpa_status dpa_route_noalloc(const dpa_layer_desc* d, const void* x, int n_tokens, const void* w_router,
                                        int32_t* topk_idx, double* topk_gate, double* logits, void* stream) {
    dpa_layer_desc probe;
    dpa_sizes sz;
    if (!d) return DPA_ERR_INVALID_ARG;
    probe = *d;
    const dpa_status st = dpa_encoded_sizes(&probe, &sz);   // validates the descriptor
    if (st != DPA_OK) return st;
    if (n_tokens <= 0 || !x || !w_router || !topk_idx || !topk_gate) return DPA_ERR_INVALID_ARG;
    if (n_tokens > kNoAllocMaxTokens || static_cast<long long>(n_tokens) * d->n_experts > kNoAllocMaxLogits)
        return DPA_ERR_UNSUPPORTED;   // beyond the fixed scratch
    auto aligned16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(topk_idx) || !aligned16(topk_gate) ||
        (logits && !aligned16(logits)))
        return DPA_ERR_INVALID_ARG;
    void* scratch = nullptr;
    if (scratch_for_current_device(&scratch) != DPA_OK) return DPA_ERR_CUDA;
    unsigned char* base = static_cast<unsigned char*>(scratch);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the per-token tickets must start at zero: clear them (and the error header) every call
    if (cudaMemsetAsync(base, 0, kCountersOff + sizeof(unsigned) * n_tokens, s) != cudaSuccess) return DPA_ERR_CUDA;
    dpa::RouteArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.wr = static_cast<const uint16_t*>(w_router);
    a.T = n_tokens;
    a.E = d->n_experts;
    a.H = d->hidden;
    a.K = d->top_k;
    a.G = d->group;
    a.norm_topk = d->norm_topk;
    a.logits_user = logits;
    a.logits_ws = reinterpret_cast<double*>(base + kLogitsOff);
    a.idx = topk_idx;
    a.gate = topk_gate;
    a.counters = reinterpret_cast<unsigned*>(base + kCountersOff);
    a.xdig = nullptr;
    a.hdr = reinterpret_cast<dpa::WsHeader*>(base);
    return dpa::launch_route(a, s) == cudaSuccess ? DPA_OK : DPA_ERR_CUDA;
}
