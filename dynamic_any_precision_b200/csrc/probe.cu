// Test support for the device-side failure handling: runs the library's bounded waits against a
// barrier that nothing completes, with a short limit, so that a test can see a wait run out and
// be reported through the workspace's error flag, while the GPU context stays usable. No copy is
// in flight and no memory outside the workspace is touched; every kernel returns after the limit.
#include <cstdint>

#include <cuda_runtime.h>

#include "common.cuh"
#include "dpa.h"

namespace dpa {
namespace {

// kind 0: the mbarrier wait of the bulk-copy and tensor-core pipelines (an arrival that never comes)
__global__ void probe_mbar_kernel(WsHeader* hdr, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait_bounded(&bar, 0, hdr, 0x7F0, limit_ns);
}

// kind 1: the abortable wait of the pipelined expert GEMV: one warp times out and sets the CTA's
// abort flag, the other warps (waiting on the same barrier) leave on the flag
__global__ void probe_abortable_kernel(WsHeader* hdr, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    // warp 0 gives up after the limit; the others would wait ten times as long but see the flag
    (void)mbar_wait_abortable(&bar, 0, &abort, hdr, 0x7F1 + (warp ? 1u : 0u), warp == 0 ? limit_ns : 10 * limit_ns);
}

// kind 2: the grid barrier of the cooperative allocation with one CTA held back (it never arrives)
__global__ void probe_grid_kernel(WsHeader* hdr, unsigned* ctr, uint64_t limit_ns) {
    __shared__ int flag;
    if (blockIdx.x == 1) return;
    (void)grid_barrier(ctr, gridDim.x, hdr, &flag, 0x7F3, limit_ns);
}

}  // namespace
}  // namespace dpa

extern "C" dpa_status dpa_debug_timeout_probe(void* ws, size_t ws_bytes, int kind, uint64_t limit_ns, void* stream) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u) || ws_bytes < 512) return DPA_ERR_INVALID_ARG;
    if (kind < 0 || kind > 2 || limit_ns < 1000u || limit_ns > 2000000000ull) return DPA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto* hdr = static_cast<dpa::WsHeader*>(ws);
    if (kind == 0) {
        dpa::probe_mbar_kernel<<<1, 32, 0, s>>>(hdr, limit_ns);
    } else if (kind == 1) {
        dpa::probe_abortable_kernel<<<1, 128, 0, s>>>(hdr, limit_ns);
    } else {
        unsigned* ctr = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(ws) + 256);
        if (cudaMemsetAsync(ctr, 0, sizeof(unsigned), s) != cudaSuccess) return DPA_ERR_CUDA;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(32);
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, dpa::probe_grid_kernel, hdr, ctr, limit_ns) != cudaSuccess) return DPA_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? DPA_OK : DPA_ERR_CUDA;
}
