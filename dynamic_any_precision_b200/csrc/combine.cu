// Gate-weighted combine of the routed experts' outputs, plus the dense always-on experts.
//
// y[t] = bf16( sum over the token's slots, in slot order, of g * o_pair  (+ shared[t]) ).
// A per-token gather (no atomics), so the sum order is fixed and the result deterministic.
// Shared experts (DeepSeekMoE-style, always on) run densely in bf16 with fp32 accumulation;
// they are neither allocated nor counted in the plane budget.
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
    const int t = blockIdx.y;
    const int n = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (n >= a.H) return;   // nothing to read or write
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
    // slots in chunks of 8: all loads of a chunk are issued before the in-order accumulation.
    // The pair positions (allocation) and gates (router) were final before the expert kernels
    // that precede this launch passed their own waits, so the first chunk's are read (from L2)
    // before this kernel's dependency wait; the per-pair outputs only after it.
    bool waited = false;
    for (int s0 = 0; s0 < a.K; s0 += 8) {
        int pos[8];
        float g[8];
        float4 o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (s0 + u < a.K) {
                pos[u] = __ldcg(a.pair_pos + t * a.K + s0 + u);
                g[u] = static_cast<float>(__ldcg(a.gate + t * a.K + s0 + u));
            }
        }
        if (!waited) {
            pdl_wait();
            waited = true;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (s0 + u < a.K) o[u] = *reinterpret_cast<const float4*>(a.out_pair + static_cast<size_t>(pos[u]) * a.H + n);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (s0 + u < a.K) {
                r.x = fmaf(g[u], o[u].x, r.x);
                r.y = fmaf(g[u], o[u].y, r.y);
                r.z = fmaf(g[u], o[u].z, r.z);
                r.w = fmaf(g[u], o[u].w, r.w);
                if (a.pair_out_user)
                    *reinterpret_cast<float4*>(a.pair_out_user + static_cast<size_t>(t * a.K + s0 + u) * a.H + n) = o[u];
            }
        }
    }
    if (!waited) pdl_wait();
    float4 acc = a.shared_out ? *reinterpret_cast<const float4*>(a.shared_out + static_cast<size_t>(t) * a.H + n)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    acc.x += r.x;
    acc.y += r.y;
    acc.z += r.z;
    acc.w += r.w;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&lo);
    packed.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(a.y + static_cast<size_t>(t) * a.H + n) = packed;
}

// ---- dense shared experts: warp per (row, expert), all tokens in chunks of 8 ----
constexpr int kTokChunk = 8;

__device__ __forceinline__ void bf16x8_to_f32(uint4 v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__global__ void __launch_bounds__(256) shared_gateup_kernel(SharedArgs a) {
    pdl_wait();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int row = warp % a.I, s = warp / a.I;
    if (s >= a.S) return;
    const uint16_t* gr = a.wg + (static_cast<size_t>(s) * a.I + row) * a.H;
    const uint16_t* ur = a.wu + (static_cast<size_t>(s) * a.I + row) * a.H;
    for (int t0 = 0; t0 < a.T; t0 += kTokChunk) {
        float ag[kTokChunk], au[kTokChunk];
#pragma unroll
        for (int i = 0; i < kTokChunk; ++i) ag[i] = au[i] = 0.f;
        for (int j = lane * 8; j < a.H; j += 256) {
            float g8[8], u8[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(gr + j), g8);
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(ur + j), u8);
#pragma unroll
            for (int i = 0; i < kTokChunk; ++i) {
                if (t0 + i < a.T) {
                    float x8[8];
                    bf16x8_to_f32(*reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0 + i) * a.H + j), x8);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        ag[i] = fmaf(g8[q], x8[q], ag[i]);
                        au[i] = fmaf(u8[q], x8[q], au[i]);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kTokChunk; ++i) {
            float g = ag[i], u = au[i];
            for (int o = 16; o > 0; o >>= 1) {
                g += __shfl_xor_sync(0xffffffffu, g, o);
                u += __shfl_xor_sync(0xffffffffu, u, o);
            }
            if (lane == 0 && t0 + i < a.T)
                a.h[(static_cast<size_t>(t0 + i) * a.S + s) * a.I + row] = g / (1.f + expf(-g)) * u;
        }
    }
}

__global__ void __launch_bounds__(256) shared_down_kernel(SharedArgs a) {
    pdl_wait();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int n = warp;
    if (n >= a.H) return;
    for (int t0 = 0; t0 < a.T; t0 += kTokChunk) {
        float acc[kTokChunk];
#pragma unroll
        for (int i = 0; i < kTokChunk; ++i) acc[i] = 0.f;
        for (int s = 0; s < a.S; ++s) {
            const uint16_t* dr = a.wd + (static_cast<size_t>(s) * a.H + n) * a.I;
            for (int j = lane * 8; j < a.I; j += 256) {
                float d8[8];
                bf16x8_to_f32(*reinterpret_cast<const uint4*>(dr + j), d8);
#pragma unroll
                for (int i = 0; i < kTokChunk; ++i) {
                    if (t0 + i < a.T) {
                        const float* hr = a.h + (static_cast<size_t>(t0 + i) * a.S + s) * a.I + j;
                        const float4 h0 = *reinterpret_cast<const float4*>(hr);
                        const float4 h1 = *reinterpret_cast<const float4*>(hr + 4);
                        acc[i] = fmaf(d8[0], h0.x, acc[i]);
                        acc[i] = fmaf(d8[1], h0.y, acc[i]);
                        acc[i] = fmaf(d8[2], h0.z, acc[i]);
                        acc[i] = fmaf(d8[3], h0.w, acc[i]);
                        acc[i] = fmaf(d8[4], h1.x, acc[i]);
                        acc[i] = fmaf(d8[5], h1.y, acc[i]);
                        acc[i] = fmaf(d8[6], h1.z, acc[i]);
                        acc[i] = fmaf(d8[7], h1.w, acc[i]);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kTokChunk; ++i) {
            float v = acc[i];
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && t0 + i < a.T) a.out[static_cast<size_t>(t0 + i) * a.H + n] = v;
        }
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
    const int per_block = 256 * 4;
    dim3 grid((a.H + per_block - 1) / per_block, a.T);
    CombineArgs b = a;
    void* args[] = {&b};
    return launch_pdl_raw(reinterpret_cast<const void*>(combine_kernel), grid, dim3(256), 0, stream, args);
}

cudaError_t launch_shared(const SharedArgs& a, cudaStream_t stream) {
    if (a.S == 0 || a.T == 0) return cudaSuccess;
    const int warps1 = a.S * a.I;
    SharedArgs b = a;
    void* args[] = {&b};
    cudaError_t err = launch_pdl_raw(reinterpret_cast<const void*>(shared_gateup_kernel), dim3((warps1 + 7) / 8),
                                     dim3(256), 0, stream, args);
    if (err != cudaSuccess) return err;
    return launch_pdl_raw(reinterpret_cast<const void*>(shared_down_kernel), dim3((a.H + 7) / 8), dim3(256), 0,
                          stream, args);
}

}  // namespace dpa
