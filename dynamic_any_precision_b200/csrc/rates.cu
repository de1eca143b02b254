// Workload-profiled per-expert read rates (DuoRate: Two-Rate Per-Expert Precision Allocation for
// MoE Serving, Abstract): one stored copy with a baked distortion tensor; online the workload's
// own prefill is profiled without labels, and a Lagrangian rate/distortion allocation under the
// decode functional is solved with one dot product per expert and a bisection. The routing
// frequency of an expert cancels from its decision and only enters the budget.
//
//   profile   m[j] = (sequential sum over tokens of x[t][j]^2) / T;  c[e] = pairs routed to e
//   D_e(k)    = <m, Tdist[e][k-1]>: 32 chunks of H/32 channels, each summed sequentially, then the
//             pairwise tree p[i] + p[i+16], + p[i+8], + p[i+4], + p[i+2], + p[i+1]
//   k_e(lam)  = argmin_k fl(D_e(k) + fl(lam * k)), ties to the smaller k
//   bisection 64 steps on [0, 2 max_e D_e(kmin) + 1]: sum_e c_e k_e(mid) > target * sum_e c_e
//             moves lo up, else hi down; the table is k_e(hi)
// Compiled with --fmad=false: every fp64 operation is one rounded IEEE operation, so the table
// matches any implementation of the same steps bit for bit.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kRateThreads = 1024;

__global__ void __launch_bounds__(256) profile_kernel(ProfileArgs a) {
    pdl_wait();
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j < a.H) {
        double acc = 0.0;
        for (int t = 0; t < a.T; ++t) {
            const double v = static_cast<double>(bf16_bits_to_float(a.x[static_cast<size_t>(t) * a.H + j]));
            acc = __dadd_rn(acc, __dmul_rn(v, v));
        }
        a.m[j] = __ddiv_rn(acc, static_cast<double>(a.T));
    }
    // pair counts per expert (zeroed by the launcher; integer adds, so the order does not matter)
    const int P = a.T * a.K;
    for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < P; p += gridDim.x * blockDim.x) {
        const int e = a.idx[p];
        if (e >= 0 && e < a.E) atomicAdd(a.counts + e, 1);
        else set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 20);
    }
}

__global__ void __launch_bounds__(kRateThreads) solve_rates_kernel(RatesArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    double* D = reinterpret_cast<double*>(smem);   // [E][nk]
    __shared__ long long s_red[kRateThreads / 32];
    __shared__ double s_mx[kRateThreads / 32];
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int nk = a.kmax - a.kmin + 1, E = a.E, H = a.H, step = H / 32;
    const double target = *a.target;
    if (!(target >= static_cast<double>(a.kmin) && target <= static_cast<double>(a.kmax))) {
        if (tid == 0) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 21);
        return;
    }
    // D_e(k): one warp per (e, k); lane c sums chunk c, then the pairwise tree
    for (int q = warp; q < E * nk; q += nw) {
        const int e = q / nk, i = q - e * nk;
        const double* t = a.tdist + (static_cast<size_t>(e) * a.B + (a.kmin + i - 1)) * H;
        double acc = 0.0;
        for (int j = lane * step; j < (lane + 1) * step; ++j) acc = __dadd_rn(acc, __dmul_rn(a.m[j], t[j]));
        for (int o = 16; o > 0; o >>= 1) {
            const double other = __shfl_down_sync(0xffffffffu, acc, o);
            if (lane < o) acc = __dadd_rn(acc, other);
        }
        if (lane == 0) D[q] = acc;
    }
    __syncthreads();
    // bracket and budget
    double mx = 0.0;
    long long csum = 0;
    for (int e = tid; e < E; e += blockDim.x) {
        mx = fmax(mx, D[e * nk]);
        csum += a.counts[e];
    }
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        csum += __shfl_xor_sync(0xffffffffu, csum, o);
    }
    if (lane == 0) { s_mx[warp] = mx; s_red[warp] = csum; }
    __syncthreads();
    mx = s_mx[0];
    csum = s_red[0];
    for (int w = 1; w < nw; ++w) { mx = fmax(mx, s_mx[w]); csum += s_red[w]; }
    __syncthreads();
    const double budget = __dmul_rn(target, static_cast<double>(csum));
    const long long nb = static_cast<long long>(floor(budget));
    double kv[4];
    for (int i = 0; i < 4; ++i) kv[i] = static_cast<double>(a.kmin + i);
    auto decide = [&](int e, double lam) {
        double best = __dadd_rn(D[e * nk], __dmul_rn(lam, kv[0]));
        int kb = a.kmin;
        for (int i = 1; i < nk; ++i) {
            const double c = __dadd_rn(D[e * nk + i], __dmul_rn(lam, kv[i]));
            if (c < best) { best = c; kb = a.kmin + i; }
        }
        return kb;
    };
    double lo = 0.0, hi = __dadd_rn(__dmul_rn(2.0, mx), 1.0);
    for (int it = 0; it < 64; ++it) {
        const double mid = __dmul_rn(0.5, __dadd_rn(lo, hi));
        long long n = 0;
        for (int e = tid; e < E; e += blockDim.x) n += static_cast<long long>(a.counts[e]) * decide(e, mid);
        for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
        if (lane == 0) s_red[warp] = n;
        __syncthreads();
        long long tot = 0;
        for (int w = 0; w < nw; ++w) tot += s_red[w];
        __syncthreads();
        if (tot > nb) lo = mid; else hi = mid;
    }
    for (int e = tid; e < E; e += blockDim.x) a.k_table[e] = static_cast<uint8_t>(decide(e, hi));
    if (tid == 0 && a.lambda_out) *a.lambda_out = hi;
}

}  // namespace

cudaError_t launch_profile(const ProfileArgs& a, cudaStream_t stream) {
    cudaError_t err = cudaMemsetAsync(a.counts, 0, sizeof(int) * a.E, stream);
    if (err != cudaSuccess) return err;
    ProfileArgs b = a;
    void* args[] = {&b};
    const int blocks = (a.H + 255) / 256;
    return launch_pdl_raw(reinterpret_cast<const void*>(profile_kernel), dim3(blocks), dim3(256), 0, stream, args);
}

size_t rates_smem_bytes(int E, int nk) { return static_cast<size_t>(E) * nk * 8; }

cudaError_t launch_solve_rates(const RatesArgs& a, cudaStream_t stream) {
    const size_t smem = rates_smem_bytes(a.E, a.kmax - a.kmin + 1);
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(solve_rates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
        if (err != cudaSuccess) return err;
    }
    RatesArgs b = a;
    void* args[] = {&b};
    return launch_pdl_raw(reinterpret_cast<const void*>(solve_rates_kernel), dim3(1), dim3(kRateThreads), smem, stream,
                          args);
}

}  // namespace dpa
