// Post-routing plane allocation and token->expert grouping.
//
// DPA-MoE, Abstract: chunks are allocated at inference time from the live router gate
// scores. DuoRate, Abstract: a Lagrangian rate-distortion allocation solved by a bisection.
// MatMoE, review "Core Contribution": a binary search sets the precision split so that the
// average bit-width meets a target.
//
// For a multiplier lambda each routed pair p (expert e, gate g) reads
//     k_p(lambda) = argmin_{kmin<=k<=kmax} fl(fl(g * r_e(k)) + fl(lambda * k))
// planes (ties to the smaller k), and N(lambda) = sum_p k_p(lambda). Exactly 64 fp64
// bisection steps on [0, 2*max_p fl(g_p r_e(kmin)) + 1] keep N(hi) <= target * P; the result
// is lambda = hi. Every fp64 operation is an explicitly rounded intrinsic and the file is
// compiled with --fmad=false, so the decisions match any IEEE implementation of these steps.
//
// Then pairs are grouped by key (expert, k): a counting sort gives each (expert, k) segment
// a contiguous range of positions; the expert GEMV reads those segments.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kAllocThreads = 1024;

__device__ __forceinline__ int choose_k(const double* c, int nk, int kmin, double lam) {
    double best = __dadd_rn(c[0], __dmul_rn(lam, static_cast<double>(kmin)));
    int kb = kmin;
    for (int i = 1; i < nk; ++i) {
        const double cost = __dadd_rn(c[i], __dmul_rn(lam, static_cast<double>(kmin + i)));
        if (cost < best) { best = cost; kb = kmin + i; }
    }
    return kb;
}

__device__ __forceinline__ int block_sum_int(int v, int* s_part, int* s_total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_part[warp] = v;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int u = lane < nw ? s_part[lane] : 0;
        for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
        if (lane == 0) *s_total = u;
    }
    __syncthreads();
    return *s_total;
}

__global__ void __launch_bounds__(kAllocThreads) allocate_kernel(AllocArgs a) {
    extern __shared__ __align__(16) int s_counts[];   // [E*nk] (permute)
    __shared__ int s_part[32];
    __shared__ int s_total;
    __shared__ double s_maxpart[32];
    __shared__ int s_ok;
    const int P = a.T * a.K;
    const int nk = a.kmax - a.kmin + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (tid == 0) {
        const double tg = *a.target;
        s_ok = (tg >= static_cast<double>(a.kmin) && tg <= static_cast<double>(a.kmax)) ? 1 : 0;
        if (!s_ok) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 10);
    }
    __syncthreads();
    int bad = 0;
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = a.idx[p];
        bad |= (e < 0 || e >= a.E) ? 1 : 0;
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0) { set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 11); s_ok = 0; }
    }
    __syncthreads();
    if (!s_ok) {
        if (a.do_permute && tid == 0) a.hdr->n_active = 0;
        return;
    }
    const double target = *a.target;

    // costs c[p][i] = fl(g_p * r_{e_p}(kmin + i))
    double mx = 0.0;
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = a.idx[p];
        const double g = a.gate[p];
        for (int i = 0; i < nk; ++i) {
            const double c = __dmul_rn(g, a.rtable[static_cast<size_t>(e) * a.B + (a.kmin + i - 1)]);
            a.cbuf[static_cast<size_t>(p) * nk + i] = c;
            if (i == 0) mx = fmax(mx, c);
        }
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_maxpart[warp] = mx;
    __syncthreads();
    mx = s_maxpart[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mx = fmax(mx, s_maxpart[w]);

    const double budget = __dmul_rn(target, static_cast<double>(P));
    double lo = 0.0;
    double hi = __dadd_rn(__dmul_rn(2.0, mx), 1.0);
    for (int it = 0; it < 64; ++it) {
        const double mid = __dmul_rn(0.5, __dadd_rn(lo, hi));
        int local = 0;
        for (int p = tid; p < P; p += blockDim.x)
            local += choose_k(a.cbuf + static_cast<size_t>(p) * nk, nk, a.kmin, mid);
        const int n = block_sum_int(local, s_part, &s_total);
        if (static_cast<double>(n) > budget) lo = mid; else hi = mid;
    }
    for (int p = tid; p < P; p += blockDim.x) {
        const int k = choose_k(a.cbuf + static_cast<size_t>(p) * nk, nk, a.kmin, hi);
        a.k_out[p] = static_cast<uint8_t>(k);
        if (a.k_copy) a.k_copy[p] = static_cast<uint8_t>(k);
    }
    if (tid == 0 && a.lambda_out) *a.lambda_out = hi;
    if (!a.do_permute) return;

    // ---------------- grouping by (expert, k) ----------------
    const int nkeys = a.E * nk;
    for (int i = tid; i < nkeys; i += blockDim.x) s_counts[i] = 0;
    __syncthreads();
    for (int p = tid; p < P; p += blockDim.x) {
        const int k = choose_k(a.cbuf + static_cast<size_t>(p) * nk, nk, a.kmin, hi);
        atomicAdd(&s_counts[a.idx[p] * nk + (k - a.kmin)], 1);
    }
    __syncthreads();
    // exclusive scan of s_counts into seg_start (each thread scans a contiguous chunk)
    const int per = (nkeys + blockDim.x - 1) / blockDim.x;
    const int k0 = tid * per, k1 = min(nkeys, k0 + per);
    int run = 0;
    for (int i = k0; i < k1; ++i) run += s_counts[i];
    // block exclusive scan of run
    int incl = run;
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_part[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int v = lane < nw ? s_part[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        s_part[lane] = v;   // inclusive per-warp totals
    }
    __syncthreads();
    int base = incl - run + (warp > 0 ? s_part[warp - 1] : 0);
    for (int i = k0; i < k1; ++i) {
        const int c = s_counts[i];
        a.seg_start[i] = base;
        s_counts[i] = base;   // becomes the placement cursor
        base += c;
    }
    if (tid == 0) a.seg_start[nkeys] = P;
    __syncthreads();
    for (int p = tid; p < P; p += blockDim.x) {
        const int k = a.k_out[p];
        const int pos = atomicAdd(&s_counts[a.idx[p] * nk + (k - a.kmin)], 1);
        a.sorted_pair[pos] = p;
        a.pair_pos[p] = pos;
    }
    __syncthreads();
    // per-expert max k and the list of active experts (ascending id)
    int act_local = 0;
    for (int e = tid; e < a.E; e += blockDim.x) {
        int km = 0;
        for (int i = 0; i < nk; ++i)
            if (a.seg_start[e * nk + i + 1] > a.seg_start[e * nk + i]) km = a.kmin + i;
        a.exp_kmax[e] = km;
        act_local += km > 0 ? 1 : 0;
    }
    // ordered compaction: experts are handled in rounds of blockDim (E <= 1024 -> one round)
    __syncthreads();
    {
        const int e = tid;
        const int flag = (e < a.E && a.exp_kmax[e] > 0) ? 1 : 0;
        int inc = flag;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        if (lane == 31) s_part[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            const int nw = blockDim.x >> 5;
            int v = lane < nw ? s_part[lane] : 0;
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            s_part[lane] = v;
        }
        __syncthreads();
        const int rank = inc - flag + (warp > 0 ? s_part[warp - 1] : 0);
        if (flag) a.active[rank] = e;
        if (tid == blockDim.x - 1) a.hdr->n_active = static_cast<uint32_t>(rank + flag);
    }
    (void)act_local;
}

}  // namespace

cudaError_t launch_allocate(const AllocArgs& a, cudaStream_t stream) {
    const int nk = a.kmax - a.kmin + 1;
    const size_t smem = static_cast<size_t>(a.E) * nk * sizeof(int);
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(allocate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
        if (err != cudaSuccess) return err;
    }
    allocate_kernel<<<1, kAllocThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace dpa
