// Variable-plane expert FFN for decode-sized batches (the hot path).
//
// Each routed pair (token t, expert e) reads only the first k planes of e's matrices
// (DPA-MoE abstract: prefix-decodable chunks; DuoRate abstract: prefix-readable weight
// stream; MatMoE review "Core Contribution": bitplane storage, floor-and-compensation).
// For uniform codes with B planes, per scale group g of a row:
//   sum_j s_g (q_hat_j - z_g) x_j = s_g [ sum_j qtrunc_j x_j + (c_k - z_g) sum_j x_j ],
//   qtrunc_j = sum_{p<k} plane_p(j) 2^(B-1-p),  c_k = (2^(B-k) - 1) / 2,
// which is the floor-and-compensation read of the first k planes. For binary-coded planes
// (b = +-1, per-plane scale alpha_p): sum_j w_j x_j = sum_{p<k} alpha_p (2 S_p - X), S_p =
// sum of x over the plane's +1 bits.
//
// Work items are (active expert, row tile). A CTA stages the item's first kmax_e planes and
// scales into shared memory with bulk copies (one mbarrier, bounded wait), then each warp:
//   - gathers bit rho of every nibble of the plane words into a register of eight 4-bit
//     codes (the plane layout puts each lane's MMA fragment in one 32-bit word per plane);
//   - masks the register into two u8 A operands (even nibbles, and odd nibbles times 16);
//   - multiplies them on the u8 x s8 MMA (m16n8k32, exact int32 accumulation) against the
//     activations held as exact fixed-point int8 digits (three per value, two tokens per n8
//     column tile);
//   - per scale group, combines the digits, applies 2^(E-22), the group scale and the
//     compensation term in fp32.
// Tokens of one expert are grouped by their plane count k; a tile of two tokens shares k, and
// tiles are processed in ascending k so the codes are built incrementally.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int NT = 4;   // n8 column tiles (two tokens each) per pass

struct TileInfo {
    int k;
    int posA, posB;   // sorted pair positions (posB = -1: empty second slot)
};

__device__ __forceinline__ int expert_tiles(const int32_t* seg, int e, int nk) {
    int n = 0;
    for (int kc = 0; kc < nk; ++kc) n += (seg[e * nk + kc + 1] - seg[e * nk + kc] + 1) >> 1;
    return n;
}

__device__ __forceinline__ TileInfo tile_info(const int32_t* seg, int e, int nk, int kmin, int tile) {
    int acc = 0;
    for (int kc = 0; kc < nk; ++kc) {
        const int s = seg[e * nk + kc];
        const int n = seg[e * nk + kc + 1] - s;
        const int nt = (n + 1) >> 1;
        if (tile < acc + nt) {
            const int i = tile - acc;
            TileInfo ti;
            ti.k = kmin + kc;
            ti.posA = s + 2 * i;
            ti.posB = (2 * i + 1 < n) ? s + 2 * i + 1 : -1;
            return ti;
        }
        acc += nt;
    }
    TileInfo ti{0, -1, -1};
    return ti;
}

// bits at nibble position rho of plane word w, moved to nibble bit t, masked
template <int RHO, int T>
__device__ __forceinline__ uint32_t nib_bits(uint32_t w) {
    uint32_t v;
    if constexpr (T >= RHO) v = w << (T - RHO);
    else v = w >> (RHO - T);
    return v & (0x11111111u << T);
}

// fp32 value of the digits a lane holds for one output row: columns 2tq, 2tq+1 of the C
// fragment are digits {0,1} (tq even) or {2, unused} (tq odd) of the token of that half.
__device__ __forceinline__ float digit_value(int lo0, int hi0, int lo1, int hi1, int tq) {
    const float c0 = static_cast<float>(lo0 + (hi0 >> 4));
    const float c1 = static_cast<float>(lo1 + (hi1 >> 4));
    return (tq & 1) ? c0 * 65536.f : fmaf(c1, 256.f, c0);
}

__device__ __forceinline__ float pow2f(int k) { return __int_as_float((k + 127) << 23); }

struct SmemSched {
    int nt;          // tiles in this pass
    TileInfo ti[NT];
    int tokA[NT], tokB[NT];
};

// ---------------------------------------------------------------------------------------
// gate + up projections, SwiGLU epilogue -> h[pos][I]
// ---------------------------------------------------------------------------------------
template <int FMT, int B>
__global__ void __launch_bounds__(kThreads) gateup_kernel(GemvArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int H = a.H, I = a.I, G = a.G;
    const int nblk = H >> 6, ng = H / G, bpg = G >> 6;
    const int nk = a.kmax - a.kmin + 1;
    const int tiles_per_expert = I >> 4;
    // shared memory carve-up
    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem);                       // [2][B][nblk][32]
    const size_t planes_bytes = static_cast<size_t>(2) * B * nblk * 128;
    unsigned char* s_meta = smem + planes_bytes;                                   // see below
    const size_t meta_bytes = FMT == DPA_FMT_UNIFORM ? static_cast<size_t>(2) * 16 * ng * 4
                                                     : static_cast<size_t>(2) * B * 16 * ng * 2;
    float* s_red = reinterpret_cast<float*>(s_meta + ((meta_bytes + 15) & ~size_t(15)));   // [4][NT][2][2][16]
    __shared__ uint64_t s_bar;
    __shared__ int s_flag;
    __shared__ SmemSched s_sched;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tq = lane & 3;
    const int n_items = static_cast<int>(a.hdr->n_active) * tiles_per_expert;
    if (threadIdx.x == 0) {
        mbar_init(&s_bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    uint32_t phase = 0;
    // this warp's scale groups
    const int g0 = (warp * ng) / kWarps, g1 = ((warp + 1) * ng) / kWarps;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int e = a.active[item / tiles_per_expert];
        const int rt = item % tiles_per_expert;
        const int kmax_e = a.exp_kmax[e];
        if (threadIdx.x == 0) {
            fence_proxy_async();   // earlier generic reads of these buffers precede the copies
            const uint32_t pbytes = static_cast<uint32_t>(nblk) * 128;
            const uint32_t mbytes = FMT == DPA_FMT_UNIFORM ? 16u * ng * 4 : 16u * ng * 2;
            const uint32_t total = 2u * kmax_e * pbytes + (FMT == DPA_FMT_UNIFORM ? 2u * mbytes : 2u * kmax_e * mbytes);
            mbar_arrive_expect_tx(&s_bar, total);
            const uint64_t plane_stride = static_cast<uint64_t>(I) * H / 8;
            for (int m = 0; m < 2; ++m) {
                const uint8_t* base = a.planes + e * a.planes_per_expert + a.planes_mat_off[m];
                for (int p = 0; p < kmax_e; ++p)
                    bulk_g2s(s_planes + (static_cast<size_t>(m * B + p) * nblk) * 32,
                             base + p * plane_stride + static_cast<uint64_t>(rt) * pbytes, pbytes, &s_bar);
                const uint8_t* mb = a.meta + e * a.meta_per_expert + a.meta_mat_off[m];
                if (FMT == DPA_FMT_UNIFORM) {
                    bulk_g2s(s_meta + m * mbytes, mb + static_cast<uint64_t>(rt) * mbytes, mbytes, &s_bar);
                } else {
                    const uint64_t mplane = static_cast<uint64_t>(I) * ng * 2;
                    for (int p = 0; p < kmax_e; ++p)
                        bulk_g2s(s_meta + (m * B + p) * mbytes, mb + p * mplane + static_cast<uint64_t>(rt) * mbytes,
                                 mbytes, &s_bar);
                }
            }
        }
        const int ntiles = expert_tiles(a.seg_start, e, nk);
        const bool ok = cta_wait_copies(&s_bar, phase, a.hdr, 100, &s_flag);
        phase ^= 1;
        if (!ok) return;

        for (int pass0 = 0; pass0 < ntiles; pass0 += NT) {
            if (threadIdx.x < NT) {
                const int i = threadIdx.x;
                if (pass0 + i < ntiles) {
                    const TileInfo ti = tile_info(a.seg_start, e, nk, a.kmin, pass0 + i);
                    s_sched.ti[i] = ti;
                    s_sched.tokA[i] = a.sorted_pair[ti.posA] / a.K;
                    s_sched.tokB[i] = ti.posB >= 0 ? a.sorted_pair[ti.posB] / a.K : -1;
                }
                if (i == 0) s_sched.nt = min(NT, ntiles - pass0);
            }
            __syncthreads();
            const int nt = s_sched.nt;
            float acc[NT][2][2];
#pragma unroll
            for (int i = 0; i < NT; ++i)
#pragma unroll
                for (int m = 0; m < 2; ++m) acc[i][m][0] = acc[i][m][1] = 0.f;
            // B-operand source rows for this lane (column n = gid: token half, digit)
            const int dig = gid & 3;
            const int half = gid >> 2;
            const int8_t* xrow[NT];
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                const int tok = half ? s_sched.tokB[i] : s_sched.tokA[i];
                xrow[i] = (i < nt && dig < 3 && tok >= 0) ? a.xdig + (static_cast<size_t>(tok) * 3 + dig) * H : nullptr;
            }
            const int my_tok_half = tq >> 1;   // C columns 2tq,2tq+1 belong to token A (tq<2) or B
            for (int g = g0; g < g1; ++g) {
                if constexpr (FMT == DPA_FMT_UNIFORM) {
                    int C[NT][2][2][4];
#pragma unroll
                    for (int i = 0; i < NT; ++i)
#pragma unroll
                        for (int m = 0; m < 2; ++m)
#pragma unroll
                            for (int h = 0; h < 2; ++h)
#pragma unroll
                                for (int r = 0; r < 4; ++r) C[i][m][h][r] = 0;
                    for (int jb = 0; jb < bpg; ++jb) {
                        const int b = g * bpg + jb;
                        uint32_t w[2][B];
#pragma unroll
                        for (int m = 0; m < 2; ++m)
#pragma unroll
                            for (int p = 0; p < B; ++p)
                                w[m][p] = p < kmax_e ? s_planes[(static_cast<size_t>(m * B + p) * nblk + b) * 32 + lane] : 0u;
                        uint32_t R[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
                        int cur = 0;
                        uint32_t Alo[2][4], Ahi[2][4];
#pragma unroll
                        for (int i = 0; i < NT; ++i) {
                            if (i < nt) {
                                const int ki = s_sched.ti[i].k;
                                if (ki > cur) {
#pragma unroll
                                    for (int p = 0; p < B; ++p) {
                                        if (p >= cur && p < ki) {
#pragma unroll
                                            for (int m = 0; m < 2; ++m) {
                                                const uint32_t wv = w[m][p];
                                                // code bit t = B-1-p
                                                switch (B - 1 - p) {
                                                    case 0: R[m][0] |= nib_bits<0, 0>(wv); R[m][1] |= nib_bits<1, 0>(wv);
                                                            R[m][2] |= nib_bits<2, 0>(wv); R[m][3] |= nib_bits<3, 0>(wv); break;
                                                    case 1: R[m][0] |= nib_bits<0, 1>(wv); R[m][1] |= nib_bits<1, 1>(wv);
                                                            R[m][2] |= nib_bits<2, 1>(wv); R[m][3] |= nib_bits<3, 1>(wv); break;
                                                    case 2: R[m][0] |= nib_bits<0, 2>(wv); R[m][1] |= nib_bits<1, 2>(wv);
                                                            R[m][2] |= nib_bits<2, 2>(wv); R[m][3] |= nib_bits<3, 2>(wv); break;
                                                    default: R[m][0] |= nib_bits<0, 3>(wv); R[m][1] |= nib_bits<1, 3>(wv);
                                                            R[m][2] |= nib_bits<2, 3>(wv); R[m][3] |= nib_bits<3, 3>(wv); break;
                                                }
                                            }
                                        }
                                    }
                                    cur = ki;
#pragma unroll
                                    for (int m = 0; m < 2; ++m)
#pragma unroll
                                        for (int r = 0; r < 4; ++r) {
                                            Alo[m][r] = R[m][r] & 0x0F0F0F0Fu;
                                            Ahi[m][r] = R[m][r] & 0xF0F0F0F0u;
                                        }
                                }
                                uint32_t b0L = 0, b1L = 0, b0H = 0, b1H = 0;
                                if (xrow[i]) {
                                    const int8_t* src = xrow[i] + 64 * b + 4 * tq;
                                    b0L = __ldg(reinterpret_cast<const uint32_t*>(src));
                                    b1L = __ldg(reinterpret_cast<const uint32_t*>(src + 16));
                                    b0H = __ldg(reinterpret_cast<const uint32_t*>(src + 32));
                                    b1H = __ldg(reinterpret_cast<const uint32_t*>(src + 48));
                                }
#pragma unroll
                                for (int m = 0; m < 2; ++m) {
                                    mma_u8s8(C[i][m][0], Alo[m][0], Alo[m][1], Alo[m][2], Alo[m][3], b0L, b1L);
                                    mma_u8s8(C[i][m][1], Ahi[m][0], Ahi[m][1], Ahi[m][2], Ahi[m][3], b0H, b1H);
                                }
                            }
                        }
                    }
                    // epilogue for group g
                    const uint32_t* meta_u = reinterpret_cast<const uint32_t*>(s_meta);
#pragma unroll
                    for (int i = 0; i < NT; ++i) {
                        if (i < nt) {
                            const int tok = my_tok_half ? s_sched.tokB[i] : s_sched.tokA[i];
                            const int ki = s_sched.ti[i].k;
                            const float ck = 0.5f * static_cast<float>((1 << (B - ki)) - 1);
                            int Eg = 0, SX = 0;
                            if (tok >= 0) { Eg = __ldg(a.xexp + tok * ng + g); SX = __ldg(a.xsum + tok * ng + g); }
                            const float sc2 = pow2f(Eg - 22);
#pragma unroll
                            for (int m = 0; m < 2; ++m) {
#pragma unroll
                                for (int rr = 0; rr < 2; ++rr) {
                                    float v = digit_value(C[i][m][0][2 * rr], C[i][m][1][2 * rr], C[i][m][0][2 * rr + 1],
                                                          C[i][m][1][2 * rr + 1], tq);
                                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                                    const int row = gid + 8 * rr;
                                    const uint32_t sz = meta_u[(m * 16 + row) * ng + g];
                                    const float s = __half2float(__ushort_as_half(static_cast<unsigned short>(sz & 0xFFFF)));
                                    const float z = __half2float(__ushort_as_half(static_cast<unsigned short>(sz >> 16)));
                                    acc[i][m][rr] = fmaf(s * sc2, fmaf(ck - z, static_cast<float>(SX), v), acc[i][m][rr]);
                                }
                            }
                        }
                    }
                } else {
                    // binary-coded planes: one MMA chain per plane, scale alpha_p per plane
                    const __half* meta_h = reinterpret_cast<const __half*>(s_meta);
#pragma unroll
                    for (int p = 0; p < B; ++p) {
                        if (p < kmax_e) {
                            int C[NT][2][2][4];
#pragma unroll
                            for (int i = 0; i < NT; ++i)
#pragma unroll
                                for (int m = 0; m < 2; ++m)
#pragma unroll
                                    for (int h = 0; h < 2; ++h)
#pragma unroll
                                        for (int r = 0; r < 4; ++r) C[i][m][h][r] = 0;
                            for (int jb = 0; jb < bpg; ++jb) {
                                const int b = g * bpg + jb;
                                uint32_t Alo[2][4], Ahi[2][4];
#pragma unroll
                                for (int m = 0; m < 2; ++m) {
                                    const uint32_t wv = s_planes[(static_cast<size_t>(m * B + p) * nblk + b) * 32 + lane];
                                    const uint32_t r0 = nib_bits<0, 0>(wv), r1 = nib_bits<1, 0>(wv);
                                    const uint32_t r2 = nib_bits<2, 0>(wv), r3 = nib_bits<3, 0>(wv);
                                    Alo[m][0] = r0 & 0x0F0F0F0Fu; Ahi[m][0] = r0 & 0xF0F0F0F0u;
                                    Alo[m][1] = r1 & 0x0F0F0F0Fu; Ahi[m][1] = r1 & 0xF0F0F0F0u;
                                    Alo[m][2] = r2 & 0x0F0F0F0Fu; Ahi[m][2] = r2 & 0xF0F0F0F0u;
                                    Alo[m][3] = r3 & 0x0F0F0F0Fu; Ahi[m][3] = r3 & 0xF0F0F0F0u;
                                }
#pragma unroll
                                for (int i = 0; i < NT; ++i) {
                                    if (i < nt && s_sched.ti[i].k > p) {
                                        uint32_t b0L = 0, b1L = 0, b0H = 0, b1H = 0;
                                        if (xrow[i]) {
                                            const int8_t* src = xrow[i] + 64 * b + 4 * tq;
                                            b0L = __ldg(reinterpret_cast<const uint32_t*>(src));
                                            b1L = __ldg(reinterpret_cast<const uint32_t*>(src + 16));
                                            b0H = __ldg(reinterpret_cast<const uint32_t*>(src + 32));
                                            b1H = __ldg(reinterpret_cast<const uint32_t*>(src + 48));
                                        }
#pragma unroll
                                        for (int m = 0; m < 2; ++m) {
                                            mma_u8s8(C[i][m][0], Alo[m][0], Alo[m][1], Alo[m][2], Alo[m][3], b0L, b1L);
                                            mma_u8s8(C[i][m][1], Ahi[m][0], Ahi[m][1], Ahi[m][2], Ahi[m][3], b0H, b1H);
                                        }
                                    }
                                }
                            }
#pragma unroll
                            for (int i = 0; i < NT; ++i) {
                                if (i < nt && s_sched.ti[i].k > p) {
                                    const int tok = my_tok_half ? s_sched.tokB[i] : s_sched.tokA[i];
                                    int Eg = 0, SX = 0;
                                    if (tok >= 0) { Eg = __ldg(a.xexp + tok * ng + g); SX = __ldg(a.xsum + tok * ng + g); }
                                    const float sc2 = pow2f(Eg - 22);
#pragma unroll
                                    for (int m = 0; m < 2; ++m) {
#pragma unroll
                                        for (int rr = 0; rr < 2; ++rr) {
                                            float v = digit_value(C[i][m][0][2 * rr], C[i][m][1][2 * rr],
                                                                  C[i][m][0][2 * rr + 1], C[i][m][1][2 * rr + 1], tq);
                                            v += __shfl_xor_sync(0xffffffffu, v, 1);
                                            const int row = gid + 8 * rr;
                                            const float al = __half2float(meta_h[((m * B + p) * 16 + row) * ng + g]);
                                            acc[i][m][rr] = fmaf(al * sc2, fmaf(2.f, v, -static_cast<float>(SX)), acc[i][m][rr]);
                                        }
                                    }
                                }
                            }
                        }
                    }
                }
            }
            // cross-warp reduction (fixed order) and SwiGLU
            if ((tq & 1) == 0) {
#pragma unroll
                for (int i = 0; i < NT; ++i)
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr)
                            s_red[((((warp * NT + i) * 2 + m) * 2 + my_tok_half) * 16) + gid + 8 * rr] = acc[i][m][rr];
            }
            __syncthreads();
            {
                const int i = threadIdx.x >> 5, tk = (threadIdx.x >> 4) & 1, row = threadIdx.x & 15;
                if (i < nt) {
                    const int pos = tk ? s_sched.ti[i].posB : s_sched.ti[i].posA;
                    if (pos >= 0) {
                        float ag = 0.f, au = 0.f;
#pragma unroll
                        for (int w = 0; w < kWarps; ++w) {
                            ag += s_red[((((w * NT + i) * 2 + 0) * 2 + tk) * 16) + row];
                            au += s_red[((((w * NT + i) * 2 + 1) * 2 + tk) * 16) + row];
                        }
                        const float hval = ag / (1.f + expf(-ag)) * au;
                        a.h[static_cast<size_t>(pos) * I + rt * 16 + row] = hval;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------------------
// down projection: out_pair[pos][H] = W_down^(k) h[pos]
// ---------------------------------------------------------------------------------------
template <int FMT, int B>
__global__ void __launch_bounds__(kThreads) down_kernel(GemvArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int H = a.H, I = a.I, G = a.G;
    const int nblk = I >> 6, ng = I / G, bpg = G >> 6;
    const int nk = a.kmax - a.kmin + 1;
    const int tiles_per_expert = H >> 6;   // 64-row items
    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem);                   // [B][4][nblk][32]
    const size_t planes_bytes = static_cast<size_t>(B) * 4 * nblk * 128;
    unsigned char* s_meta = smem + planes_bytes;
    const size_t meta_bytes = FMT == DPA_FMT_UNIFORM ? static_cast<size_t>(64) * ng * 4
                                                     : static_cast<size_t>(B) * 64 * ng * 2;
    int8_t* s_dig = reinterpret_cast<int8_t*>(s_meta + ((meta_bytes + 15) & ~size_t(15)));   // [2NT][3][I]
    int* s_exp = reinterpret_cast<int*>(s_dig + static_cast<size_t>(2 * NT) * 3 * I);          // [2NT][ng]
    int* s_sum = s_exp + 2 * NT * ng;
    __shared__ uint64_t s_bar;
    __shared__ int s_flag;
    __shared__ SmemSched s_sched;
    __shared__ int s_pos[2 * NT];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tq = lane & 3;
    const int n_items = static_cast<int>(a.hdr->n_active) * tiles_per_expert;
    if (threadIdx.x == 0) {
        mbar_init(&s_bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    uint32_t phase = 0;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int e = a.active[item / tiles_per_expert];
        const int rt = item % tiles_per_expert;
        const int kmax_e = a.exp_kmax[e];
        if (threadIdx.x == 0) {
            fence_proxy_async();
            const uint32_t pbytes = 4u * nblk * 128;
            const uint32_t mbytes = FMT == DPA_FMT_UNIFORM ? 64u * ng * 4 : 64u * ng * 2;
            const uint32_t total = kmax_e * pbytes + (FMT == DPA_FMT_UNIFORM ? mbytes : kmax_e * mbytes);
            mbar_arrive_expect_tx(&s_bar, total);
            const uint64_t plane_stride = static_cast<uint64_t>(H) * I / 8;
            const uint8_t* base = a.planes + e * a.planes_per_expert + a.planes_mat_off[2];
            for (int p = 0; p < kmax_e; ++p)
                bulk_g2s(s_planes + static_cast<size_t>(p) * 4 * nblk * 32,
                         base + p * plane_stride + static_cast<uint64_t>(rt) * pbytes, pbytes, &s_bar);
            const uint8_t* mb = a.meta + e * a.meta_per_expert + a.meta_mat_off[2];
            if (FMT == DPA_FMT_UNIFORM) {
                bulk_g2s(s_meta, mb + static_cast<uint64_t>(rt) * mbytes, mbytes, &s_bar);
            } else {
                const uint64_t mplane = static_cast<uint64_t>(H) * ng * 2;
                for (int p = 0; p < kmax_e; ++p)
                    bulk_g2s(s_meta + p * mbytes, mb + p * mplane + static_cast<uint64_t>(rt) * mbytes, mbytes, &s_bar);
            }
        }
        const int ntiles = expert_tiles(a.seg_start, e, nk);
        bool copied = false;

        for (int pass0 = 0; pass0 < ntiles; pass0 += NT) {
            if (threadIdx.x < NT) {
                const int i = threadIdx.x;
                if (pass0 + i < ntiles) {
                    const TileInfo ti = tile_info(a.seg_start, e, nk, a.kmin, pass0 + i);
                    s_sched.ti[i] = ti;
                    s_pos[2 * i] = ti.posA;
                    s_pos[2 * i + 1] = ti.posB;
                } else {
                    s_pos[2 * i] = -1;
                    s_pos[2 * i + 1] = -1;
                }
                if (i == 0) s_sched.nt = min(NT, ntiles - pass0);
            }
            __syncthreads();
            const int nt = s_sched.nt;
            // fixed-point digits of the pass's h rows: one warp per (slot, group)
            for (int task = warp; task < 2 * NT * ng; task += kWarps) {
                const int slot = task / ng, g = task % ng;
                const int pos = s_pos[slot];
                if (pos < 0) continue;
                const float* hrow = a.h + static_cast<size_t>(pos) * I + g * G;
                float mx = 0.f;
                for (int j = lane; j < G; j += 32) mx = fmaxf(mx, fabsf(hrow[j]));
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const int Eg = group_exponent(mx);
                int sum = 0;
                for (int j = lane; j < G; j += 32) {
                    const int X = to_fixed(hrow[j], Eg);
                    sum += X;
                    int8_t d0, d1, d2;
                    split_digits(X, d0, d1, d2);
                    int8_t* dst = s_dig + static_cast<size_t>(slot) * 3 * I + g * G + j;
                    dst[0] = d0;
                    dst[I] = d1;
                    dst[2 * I] = d2;
                }
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) { s_exp[slot * ng + g] = Eg; s_sum[slot * ng + g] = sum; }
            }
            if (!copied) {
                const bool ok = cta_wait_copies(&s_bar, phase, a.hdr, 200, &s_flag);
                phase ^= 1;
                copied = true;
                if (!ok) return;
            }
            __syncthreads();

            float acc[NT][2];
#pragma unroll
            for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = 0.f;
            const int dig = gid & 3, half = gid >> 2;
            const int8_t* xrow[NT];
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                const int slot = 2 * i + half;
                xrow[i] = (i < nt && dig < 3 && s_pos[slot] >= 0) ? s_dig + (static_cast<size_t>(slot) * 3 + dig) * I : nullptr;
            }
            const int my_half = tq >> 1;
            const uint32_t* wplanes = s_planes + static_cast<size_t>(warp) * nblk * 32;   // tile `warp` of 4
            for (int g = 0; g < ng; ++g) {
                if constexpr (FMT == DPA_FMT_UNIFORM) {
                    int C[NT][2][4];
#pragma unroll
                    for (int i = 0; i < NT; ++i)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int r = 0; r < 4; ++r) C[i][h][r] = 0;
                    for (int jb = 0; jb < bpg; ++jb) {
                        const int b = g * bpg + jb;
                        uint32_t w[B];
#pragma unroll
                        for (int p = 0; p < B; ++p)
                            w[p] = p < kmax_e ? wplanes[(static_cast<size_t>(p) * 4 * nblk + b) * 32 + lane] : 0u;
                        uint32_t R[4] = {0u, 0u, 0u, 0u};
                        int cur = 0;
                        uint32_t Alo[4], Ahi[4];
#pragma unroll
                        for (int i = 0; i < NT; ++i) {
                            if (i < nt) {
                                const int ki = s_sched.ti[i].k;
                                if (ki > cur) {
#pragma unroll
                                    for (int p = 0; p < B; ++p) {
                                        if (p >= cur && p < ki) {
                                            const uint32_t wv = w[p];
                                            switch (B - 1 - p) {
                                                case 0: R[0] |= nib_bits<0, 0>(wv); R[1] |= nib_bits<1, 0>(wv);
                                                        R[2] |= nib_bits<2, 0>(wv); R[3] |= nib_bits<3, 0>(wv); break;
                                                case 1: R[0] |= nib_bits<0, 1>(wv); R[1] |= nib_bits<1, 1>(wv);
                                                        R[2] |= nib_bits<2, 1>(wv); R[3] |= nib_bits<3, 1>(wv); break;
                                                case 2: R[0] |= nib_bits<0, 2>(wv); R[1] |= nib_bits<1, 2>(wv);
                                                        R[2] |= nib_bits<2, 2>(wv); R[3] |= nib_bits<3, 2>(wv); break;
                                                default: R[0] |= nib_bits<0, 3>(wv); R[1] |= nib_bits<1, 3>(wv);
                                                        R[2] |= nib_bits<2, 3>(wv); R[3] |= nib_bits<3, 3>(wv); break;
                                            }
                                        }
                                    }
                                    cur = ki;
#pragma unroll
                                    for (int r = 0; r < 4; ++r) {
                                        Alo[r] = R[r] & 0x0F0F0F0Fu;
                                        Ahi[r] = R[r] & 0xF0F0F0F0u;
                                    }
                                }
                                uint32_t b0L = 0, b1L = 0, b0H = 0, b1H = 0;
                                if (xrow[i]) {
                                    const int8_t* src = xrow[i] + 64 * b + 4 * tq;
                                    b0L = *reinterpret_cast<const uint32_t*>(src);
                                    b1L = *reinterpret_cast<const uint32_t*>(src + 16);
                                    b0H = *reinterpret_cast<const uint32_t*>(src + 32);
                                    b1H = *reinterpret_cast<const uint32_t*>(src + 48);
                                }
                                mma_u8s8(C[i][0], Alo[0], Alo[1], Alo[2], Alo[3], b0L, b1L);
                                mma_u8s8(C[i][1], Ahi[0], Ahi[1], Ahi[2], Ahi[3], b0H, b1H);
                            }
                        }
                    }
                    const uint32_t* meta_u = reinterpret_cast<const uint32_t*>(s_meta);
#pragma unroll
                    for (int i = 0; i < NT; ++i) {
                        if (i < nt) {
                            const int slot = 2 * i + my_half;
                            const int ki = s_sched.ti[i].k;
                            const float ck = 0.5f * static_cast<float>((1 << (B - ki)) - 1);
                            const int Eg = s_exp[slot * ng + g], SX = s_sum[slot * ng + g];
                            const float sc2 = pow2f(Eg - 22);
#pragma unroll
                            for (int rr = 0; rr < 2; ++rr) {
                                float v = digit_value(C[i][0][2 * rr], C[i][1][2 * rr], C[i][0][2 * rr + 1], C[i][1][2 * rr + 1], tq);
                                v += __shfl_xor_sync(0xffffffffu, v, 1);
                                const int row = warp * 16 + gid + 8 * rr;
                                const uint32_t sz = meta_u[row * ng + g];
                                const float s = __half2float(__ushort_as_half(static_cast<unsigned short>(sz & 0xFFFF)));
                                const float z = __half2float(__ushort_as_half(static_cast<unsigned short>(sz >> 16)));
                                acc[i][rr] = fmaf(s * sc2, fmaf(ck - z, static_cast<float>(SX), v), acc[i][rr]);
                            }
                        }
                    }
                } else {
                    const __half* meta_h = reinterpret_cast<const __half*>(s_meta);
#pragma unroll
                    for (int p = 0; p < B; ++p) {
                        if (p < kmax_e) {
                            int C[NT][2][4];
#pragma unroll
                            for (int i = 0; i < NT; ++i)
#pragma unroll
                                for (int h = 0; h < 2; ++h)
#pragma unroll
                                    for (int r = 0; r < 4; ++r) C[i][h][r] = 0;
                            for (int jb = 0; jb < bpg; ++jb) {
                                const int b = g * bpg + jb;
                                const uint32_t wv = wplanes[(static_cast<size_t>(p) * 4 * nblk + b) * 32 + lane];
                                const uint32_t r0 = nib_bits<0, 0>(wv), r1 = nib_bits<1, 0>(wv);
                                const uint32_t r2 = nib_bits<2, 0>(wv), r3 = nib_bits<3, 0>(wv);
                                const uint32_t Alo[4] = {r0 & 0x0F0F0F0Fu, r1 & 0x0F0F0F0Fu, r2 & 0x0F0F0F0Fu, r3 & 0x0F0F0F0Fu};
                                const uint32_t Ahi[4] = {r0 & 0xF0F0F0F0u, r1 & 0xF0F0F0F0u, r2 & 0xF0F0F0F0u, r3 & 0xF0F0F0F0u};
#pragma unroll
                                for (int i = 0; i < NT; ++i) {
                                    if (i < nt && s_sched.ti[i].k > p) {
                                        uint32_t b0L = 0, b1L = 0, b0H = 0, b1H = 0;
                                        if (xrow[i]) {
                                            const int8_t* src = xrow[i] + 64 * b + 4 * tq;
                                            b0L = *reinterpret_cast<const uint32_t*>(src);
                                            b1L = *reinterpret_cast<const uint32_t*>(src + 16);
                                            b0H = *reinterpret_cast<const uint32_t*>(src + 32);
                                            b1H = *reinterpret_cast<const uint32_t*>(src + 48);
                                        }
                                        mma_u8s8(C[i][0], Alo[0], Alo[1], Alo[2], Alo[3], b0L, b1L);
                                        mma_u8s8(C[i][1], Ahi[0], Ahi[1], Ahi[2], Ahi[3], b0H, b1H);
                                    }
                                }
                            }
#pragma unroll
                            for (int i = 0; i < NT; ++i) {
                                if (i < nt && s_sched.ti[i].k > p) {
                                    const int slot = 2 * i + my_half;
                                    const int Eg = s_exp[slot * ng + g], SX = s_sum[slot * ng + g];
                                    const float sc2 = pow2f(Eg - 22);
#pragma unroll
                                    for (int rr = 0; rr < 2; ++rr) {
                                        float v = digit_value(C[i][0][2 * rr], C[i][1][2 * rr], C[i][0][2 * rr + 1],
                                                              C[i][1][2 * rr + 1], tq);
                                        v += __shfl_xor_sync(0xffffffffu, v, 1);
                                        const int row = warp * 16 + gid + 8 * rr;
                                        const float al = __half2float(meta_h[(p * 64 + row) * ng + g]);
                                        acc[i][rr] = fmaf(al * sc2, fmaf(2.f, v, -static_cast<float>(SX)), acc[i][rr]);
                                    }
                                }
                            }
                        }
                    }
                }
            }
            // write outputs: lanes tq = 0 (token A) and tq = 2 (token B)
            if ((tq & 1) == 0) {
#pragma unroll
                for (int i = 0; i < NT; ++i) {
                    if (i < nt) {
                        const int pos = s_pos[2 * i + my_half];
                        if (pos >= 0) {
#pragma unroll
                            for (int rr = 0; rr < 2; ++rr)
                                a.out_pair[static_cast<size_t>(pos) * H + rt * 64 + warp * 16 + gid + 8 * rr] = acc[i][rr];
                        }
                    }
                }
            }
            __syncthreads();
        }
        if (!copied) {   // expert without tiles cannot happen (active), but keep the phase right
            const bool ok = cta_wait_copies(&s_bar, phase, a.hdr, 202, &s_flag);
            phase ^= 1;
            if (!ok) return;
        }
        __syncthreads();
    }
}

template <int FMT>
void* pick_gateup(int B) {
    switch (B) {
        case 1: return reinterpret_cast<void*>(gateup_kernel<FMT, 1>);
        case 2: return reinterpret_cast<void*>(gateup_kernel<FMT, 2>);
        case 3: return reinterpret_cast<void*>(gateup_kernel<FMT, 3>);
        default: return reinterpret_cast<void*>(gateup_kernel<FMT, 4>);
    }
}
template <int FMT>
void* pick_down(int B) {
    switch (B) {
        case 1: return reinterpret_cast<void*>(down_kernel<FMT, 1>);
        case 2: return reinterpret_cast<void*>(down_kernel<FMT, 2>);
        case 3: return reinterpret_cast<void*>(down_kernel<FMT, 3>);
        default: return reinterpret_cast<void*>(down_kernel<FMT, 4>);
    }
}

}  // namespace

size_t gateup_smem_bytes(const GemvArgs& a) {
    const int nblk = a.H >> 6, ng = a.H / a.G;
    size_t planes = static_cast<size_t>(2) * a.B * nblk * 128;
    size_t meta = a.fmt == DPA_FMT_UNIFORM ? static_cast<size_t>(2) * 16 * ng * 4 : static_cast<size_t>(2) * a.B * 16 * ng * 2;
    meta = (meta + 15) & ~size_t(15);
    return planes + meta + static_cast<size_t>(kWarps) * NT * 2 * 2 * 16 * 4;
}

size_t down_smem_bytes(const GemvArgs& a) {
    const int nblk = a.I >> 6, ng = a.I / a.G;
    size_t planes = static_cast<size_t>(a.B) * 4 * nblk * 128;
    size_t meta = a.fmt == DPA_FMT_UNIFORM ? static_cast<size_t>(64) * ng * 4 : static_cast<size_t>(a.B) * 64 * ng * 2;
    meta = (meta + 15) & ~size_t(15);
    return planes + meta + static_cast<size_t>(2 * NT) * 3 * a.I + static_cast<size_t>(2 * NT) * ng * 8;
}

static cudaError_t launch_generic(void* fn, size_t smem, int grid, const GemvArgs& a, cudaStream_t stream) {
    if (grid <= 0) return cudaSuccess;
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    GemvArgs copy = a;
    void* args[] = {&copy};
    return cudaLaunchKernel(fn, dim3(grid), dim3(kThreads), args, smem, stream);
}

cudaError_t launch_gateup(const GemvArgs& a, cudaStream_t stream, int num_sms) {
    void* fn = a.fmt == DPA_FMT_UNIFORM ? pick_gateup<DPA_FMT_UNIFORM>(a.B) : pick_gateup<DPA_FMT_BCQ>(a.B);
    const int items = a.max_items * (a.I >> 4);
    const int grid = items < num_sms * 4 ? items : num_sms * 4;
    return launch_generic(fn, gateup_smem_bytes(a), grid, a, stream);
}

cudaError_t launch_down(const GemvArgs& a, cudaStream_t stream, int num_sms) {
    void* fn = a.fmt == DPA_FMT_UNIFORM ? pick_down<DPA_FMT_UNIFORM>(a.B) : pick_down<DPA_FMT_BCQ>(a.B);
    const int items = a.max_items * (a.H >> 6);
    const int grid = items < num_sms * 4 ? items : num_sms * 4;
    return launch_generic(fn, down_smem_bytes(a), grid, a, stream);
}

}  // namespace dpa
