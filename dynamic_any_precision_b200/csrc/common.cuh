// Device helpers shared by the sm_100a kernels: workspace header, error flag, bounded
// mbarrier waits, bulk global->shared copies, MMA wrappers.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dpa.h"

namespace dpa {

// Tokens per tile of the prefill tensor-core GEMMs (the MMA's N extent at most).
constexpr int kGemmTileTokens = 128;

// ---- workspace header (first 256 bytes of every workspace) ----
struct WsHeader {
    uint32_t error;       // first device error code (0 = none)
    uint32_t error_info;  // kernel-specific detail (which wait, which index)
    uint32_t n_active;    // routed experts with at least one pair in the last forward
    uint32_t n_gtiles;    // token tiles of the prefill GEMMs in the last forward (0 on the decode path)
    uint32_t n_vgroups;   // token groups of the pipelined expert GEMV in the last forward
    uint32_t pad[59];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte block");

__device__ __forceinline__ void set_error(WsHeader* h, uint32_t code, uint32_t info) {
    if (atomicCAS(&h->error, 0u, code) == 0u) h->error_info = info;
}

// ---- bounded waits ----
// Every spin in these kernels gives up after kWaitNs nanoseconds (device clock), records
// DPA_ERR_DEVICE_TIMEOUT and returns, so a lost completion can never hang the GPU.
constexpr uint64_t kWaitNs = 200ull * 1000ull * 1000ull;   // 200 ms

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbarrier_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended (not spinning, so issuing nothing) for up to
// `ns` nanoseconds while the phase is incomplete.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` with a time limit. Returns false on timeout (after
// recording the error). The caller must not read the buffers the barrier guards then.
// While waiting, the thread sleeps in the barrier for up to 20 us per try instead of spinning.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, WsHeader* hdr,
                                                  uint32_t where, uint64_t limit_ns = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait_suspend(bar, parity, 20000u)) {
        if (globaltimer() - t0 > limit_ns) {
            set_error(hdr, DPA_ERR_DEVICE_TIMEOUT, where);
            return false;
        }
    }
    return true;
}

// The same wait for kernels whose roles end together: it also gives up as soon as another thread
// of the CTA has set `abort` (after a timeout of its own), and a timeout sets `abort`.
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                    WsHeader* hdr, uint32_t where, uint64_t limit_ns = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait_suspend(bar, parity, 10000u)) {
        if (*abort) return false;
        if (globaltimer() - t0 > limit_ns) {
            set_error(hdr, DPA_ERR_DEVICE_TIMEOUT, where);
            *abort = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid barrier of a cooperatively launched (hence co-resident) grid: every CTA adds one to *ctr
// and waits until it reaches `target`; false (and DPA_ERR_DEVICE_TIMEOUT recorded) when the
// limit runs out first. The verdict is shared with the CTA through *s_flag.
__device__ __forceinline__ bool grid_barrier(unsigned* ctr, unsigned target, WsHeader* hdr, int* s_flag,
                                             uint32_t where = 0x240, uint64_t limit_ns = kWaitNs) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);
        bool ok = true;
        if (ld_acquire_u32(ctr) < target) {
            const uint64_t t0 = globaltimer();
            while (ld_acquire_u32(ctr) < target) {
                if (globaltimer() - t0 > limit_ns) {
                    set_error(hdr, DPA_ERR_DEVICE_TIMEOUT, where);
                    ok = false;
                    break;
                }
            }
        }
        *s_flag = ok ? 1 : 0;
    }
    __syncthreads();
    return *s_flag != 0;
}

// CTA-uniform wait for a bulk-copy phase: thread 0 waits with a time limit (and on a
// timeout gives the copies a second bounded chance to land, so none is left writing into
// shared memory of a CTA that exits); the verdict is broadcast through `flag` so that every
// thread returns or continues together. Then each thread observes the completed phase
// itself (immediate), which orders the copied data before its reads.
__device__ __forceinline__ bool cta_wait_copies(uint64_t* bar, uint32_t parity, WsHeader* hdr, uint32_t where,
                                                int* flag) {
    if (threadIdx.x == 0) {
        bool ok = mbar_wait_bounded(bar, parity, hdr, where);
        if (!ok) mbar_wait_bounded(bar, parity, hdr, where + 1);
        *flag = ok ? 1 : 0;
    }
    __syncthreads();
    const bool ok = *flag != 0;
    if (ok) (void)mbar_try_wait(bar, parity);
    return ok;
}

// Order this thread's (and, after a barrier, the CTA's) generic-proxy shared-memory accesses
// before later async-proxy (bulk copy) writes to the same buffers.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- thread-block clusters: rank, distributed shared memory, cluster-scope mbarriers ----
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// address of the same shared-memory object in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}
// asynchronous remote store of 4 bytes into CTA shared memory of the cluster that completes 4
// bytes of transaction count on that CTA's mbarrier (both shared::cluster addresses)
__device__ __forceinline__ void st_async_s32(uint32_t cluster_addr, int v, uint32_t cluster_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(cluster_addr),
                 "r"(v), "r"(cluster_bar)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// the cluster's mbarrier initialisations become visible to the other CTAs
__device__ __forceinline__ void fence_mbarrier_init_cluster() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// hardware barrier of the whole cluster (used once, right after the mbarrier initialisation,
// when every CTA of the cluster is resident by construction)
__device__ __forceinline__ void cluster_barrier_once() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Untiled bulk copy global -> shared, completing `bytes` of transaction count on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16. No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---- programmatic dependent launch ----
// Kernels of a forward are launched with programmatic stream serialisation. A successor is
// released when every CTA of its predecessor has triggered or exited; the launch and prologue
// work before wait (descriptor and weight prefetch) then overlap the predecessor. wait blocks
// until the predecessor has completed and its memory is visible; every kernel calls it before
// its first read of a predecessor's output and before its first global write. Outside such a
// launch both are no-ops. The single-CTA allocation and the gate/up kernel trigger early
// (after their own waits): the next kernel's CTAs then become resident and read what is
// already final (work lists, static weights) while the predecessor runs. (Triggering in every
// kernel was measured slower at batch 1, 42.9 vs 41.1 us per step: early-resident successor
// CTAs take SM slots from a wide predecessor.)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with programmatic stream serialisation (see above).
inline cudaError_t launch_pdl_raw(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                  void** args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

// ---- u8 x s8 MMA, m16n8k32, int32 accumulate ----
__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- fixed-point digits of a group of activations ----
// A group of values v_j is represented exactly (or to 22 fractional bits of its largest
// magnitude) as v_j = X_j * 2^(E - 22) with |X_j| <= 2^22, E = exponent with max|v| < 2^E.
// X_j is split into balanced base-256 digits d0 + 256*d1 + 65536*d2, each an int8, which are
// the s8 operand of the MMA.
__device__ __forceinline__ int group_exponent(float maxabs) {
    if (!(maxabs > 0.f)) return 0;
    int e;
    frexpf(maxabs, &e);
    return e;
}

__device__ __forceinline__ int to_fixed(float v, int E) {
    return __float2int_rn(ldexpf(v, 22 - E));
}

__device__ __forceinline__ void split_digits(int X, int8_t& d0, int8_t& d1, int8_t& d2) {
    const int a0 = ((X + 128) & 255) - 128;
    const int X1 = (X - a0) >> 8;
    const int a1 = ((X1 + 128) & 255) - 128;
    const int a2 = (X1 - a1) >> 8;
    d0 = static_cast<int8_t>(a0);
    d1 = static_cast<int8_t>(a1);
    d2 = static_cast<int8_t>(a2);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

}  // namespace dpa
