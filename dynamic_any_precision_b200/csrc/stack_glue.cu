// Glue between the MoE layers of a stack (pre-norm residual; the pages give no form, and
// this is the plainest reading of "residual add and RMSNorm between layers"):
//     h <- h + y            (fp32 residual stream; skipped when y is NULL)
//     x <- bf16( h / sqrt(mean(h^2) + eps) )
// One CTA per token. The mean of squares is accumulated in fp32 per thread, then reduced in a
// fixed order (warp butterflies, then warps in order), so the result is deterministic.
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kGlueThreads = 256;

__global__ void __launch_bounds__(kGlueThreads) residual_rmsnorm_kernel(const uint16_t* y, float* h, uint16_t* x,
                                                                         int H, float eps) {
    __shared__ float s_part[kGlueThreads / 32];
    pdl_wait();
    const int t = blockIdx.x;
    float* hr = h + static_cast<size_t>(t) * H;
    const uint16_t* yr = y ? y + static_cast<size_t>(t) * H : nullptr;
    float ss = 0.f;
    for (int j = threadIdx.x * 4; j < H; j += kGlueThreads * 4) {
        float4 v = *reinterpret_cast<const float4*>(hr + j);
        if (yr) {
            const uint2 yy = *reinterpret_cast<const uint2*>(yr + j);
            v.x += __uint_as_float(yy.x << 16);
            v.y += __uint_as_float(yy.x & 0xFFFF0000u);
            v.z += __uint_as_float(yy.y << 16);
            v.w += __uint_as_float(yy.y & 0xFFFF0000u);
            *reinterpret_cast<float4*>(hr + j) = v;
        }
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
    }
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kGlueThreads / 32; ++w) tot += s_part[w];
    const float inv = rsqrtf(tot / static_cast<float>(H) + eps);
    uint16_t* xr = x + static_cast<size_t>(t) * H;
    for (int j = threadIdx.x * 4; j < H; j += kGlueThreads * 4) {
        const float4 v = *reinterpret_cast<const float4*>(hr + j);
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x * inv, v.y * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(v.z * inv, v.w * inv);
        uint2 packed;
        packed.x = *reinterpret_cast<uint32_t*>(&lo);
        packed.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(xr + j) = packed;
    }
}

}  // namespace

cudaError_t launch_residual_rmsnorm(const uint16_t* y, float* h, uint16_t* x, int T, int H, float eps,
                                    cudaStream_t stream) {
    void* args[] = {&y, &h, &x, &H, &eps};
    return launch_pdl_raw(reinterpret_cast<const void*>(residual_rmsnorm_kernel), dim3(T), dim3(kGlueThreads), 0, stream,
                          args);
}

}  // namespace dpa
