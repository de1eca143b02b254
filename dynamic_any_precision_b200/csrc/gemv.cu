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
// scales into shared memory with bulk copies (one mbarrier, bounded wait) and the
// activations' fixed-point digits with vector loads, then each warp:
//   - gathers bit rho of every nibble of the plane words into a register of eight 4-bit
//     codes (the plane layout puts each lane's MMA fragment in one 32-bit word per plane);
//   - masks the register into two u8 A operands (even nibbles, and odd nibbles times 16);
//   - multiplies them on the u8 x s8 MMA (m16n8k32, exact int32 accumulation) against the
//     activations held as exact fixed-point int8 digits (three per value, two tokens per n8
//     column tile);
//   - per scale group, combines the digits, applies 2^(E-22), the group scale and the
//     compensation term in fp32.
// Tokens of one expert are grouped by their plane count k; a tile of two tokens shares k, and
// tiles come in ascending k so the codes are built incrementally.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kDigPad = 16;   // bytes added to each digit row in shared memory (bank spread)

// bits at nibble position rho of plane word w, moved to nibble bit t, masked
template <int RHO, int T>
__device__ __forceinline__ uint32_t nib_bits(uint32_t w) {
    uint32_t v;
    if constexpr (T >= RHO) v = w << (T - RHO);
    else v = w >> (RHO - T);
    return v & (0x11111111u << T);
}

// OR the bits of plane word w (code bit t) into the four nibble registers
template <int T>
__device__ __forceinline__ void add_plane(uint32_t (&R)[4], uint32_t w) {
    R[0] |= nib_bits<0, T>(w);
    R[1] |= nib_bits<1, T>(w);
    R[2] |= nib_bits<2, T>(w);
    R[3] |= nib_bits<3, T>(w);
}

// OR planes [FROM, TO) (plane p at pl[p * ps]) into the nibble registers; code bit = B-1-p
template <int B, int FROM, int TO>
__device__ __forceinline__ void add_range(uint32_t (&R)[4], const uint32_t* pl, int ps) {
    if constexpr (FROM < TO && FROM < B) {
        add_plane<B - 1 - FROM>(R, pl[FROM * ps]);
        add_range<B, FROM + 1, TO>(R, pl, ps);
    }
}

// planes [from, to) with a warp-uniform jump: only the planes a tile reads are loaded and merged
template <int B>
__device__ __forceinline__ void add_planes(uint32_t (&R)[4], const uint32_t* pl, int ps, int from, int to) {
    switch (from * 5 + to) {
        case 1: add_range<B, 0, 1>(R, pl, ps); break;
        case 2: add_range<B, 0, 2>(R, pl, ps); break;
        case 3: add_range<B, 0, 3>(R, pl, ps); break;
        case 4: add_range<B, 0, 4>(R, pl, ps); break;
        case 7: add_range<B, 1, 2>(R, pl, ps); break;
        case 8: add_range<B, 1, 3>(R, pl, ps); break;
        case 9: add_range<B, 1, 4>(R, pl, ps); break;
        case 13: add_range<B, 2, 3>(R, pl, ps); break;
        case 14: add_range<B, 2, 4>(R, pl, ps); break;
        case 19: add_range<B, 3, 4>(R, pl, ps); break;
        default: break;
    }
}

// fp32 value of the digits a lane holds for one output row: columns 2tq, 2tq+1 of the C
// fragment are digits {0,1} (tq even) or {2, unused} (tq odd) of the token of that half.
__device__ __forceinline__ float digit_value(int lo0, int hi0, int lo1, int hi1, int tq) {
    const float c0 = static_cast<float>(lo0 + (hi0 >> 4));
    const float c1 = static_cast<float>(lo1 + (hi1 >> 4));
    return (tq & 1) ? c0 * 65536.f : fmaf(c1, 256.f, c0);
}

__device__ __forceinline__ float pow2f(int k) { return __int_as_float((k + 127) << 23); }

__device__ __forceinline__ int tile_tok(const int4& t, int half) {
    const int v = half ? (t.w >> 16) & 0xFFFF : t.w & 0xFFFF;
    return v == 0xFFFF ? -1 : v;
}

__device__ __forceinline__ void load_b(const int8_t* row, int b, int tq, uint32_t& b0L, uint32_t& b1L,
                                       uint32_t& b0H, uint32_t& b1H) {
    const int8_t* src = row + 64 * b + 4 * tq;
    b0L = *reinterpret_cast<const uint32_t*>(src);
    b1L = *reinterpret_cast<const uint32_t*>(src + 16);
    b0H = *reinterpret_cast<const uint32_t*>(src + 32);
    b1H = *reinterpret_cast<const uint32_t*>(src + 48);
}


// Bulk copies (no multicast) of one pass's activation digits into the padded shared slots:
// lane s of warp 0 (s < 2 NT) copies the three W-byte digit rows of its slot's source row
// src (a token, or a pair position) and, when copy_es, its ng exponents and sums. Empty slots
// get zero exponents and sums. One arrive with the total byte count completes the barrier.
template <int NT>
__device__ __forceinline__ void issue_digit_copies(int src, const int8_t* dig, const int32_t* ex, const int32_t* sm, int W,
                                                   int ng, bool copy_es, int8_t* s_dig, int dstride, int* s_xe, int* s_xs,
                                                   uint64_t* bar) {
    const int lane = threadIdx.x & 31;
    const unsigned valid = __ballot_sync(0xffffffffu, lane < 2 * NT && src >= 0);
    if (lane == 0) {
        const uint32_t per = 3u * static_cast<uint32_t>(W) + (copy_es ? 8u * static_cast<uint32_t>(ng) : 0u);
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(__popc(valid)) * per);
    }
    __syncwarp();
    if (lane < 2 * NT) {
        if (src >= 0) {
            fence_proxy_async();   // the CTA's earlier generic reads of the slot precede the copies
            const int8_t* row = dig + static_cast<size_t>(src) * 3 * W;
            for (int d = 0; d < 3; ++d) bulk_g2s(s_dig + (lane * 3 + d) * dstride, row + d * W, static_cast<uint32_t>(W), bar);
            if (copy_es) {
                bulk_g2s(s_xe + lane * ng, ex + static_cast<size_t>(src) * ng, static_cast<uint32_t>(ng) * 4u, bar);
                bulk_g2s(s_xs + lane * ng, sm + static_cast<size_t>(src) * ng, static_cast<uint32_t>(ng) * 4u, bar);
            }
        } else if (copy_es) {
            for (int g = 0; g < ng; ++g) { s_xe[lane * ng + g] = 0; s_xs[lane * ng + g] = 0; }
        }
    }
}

struct Layout {
    // byte offsets inside dynamic shared memory
    size_t planes, meta, dig, xe, xs, red, total;
    int dig_stride;   // bytes per digit row
};

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~static_cast<size_t>(15); }

// gate/up: planes [2][B][nblk][32], meta, digits [2NT][3][H+pad], exps/sums [2NT][ng], red
__host__ __device__ inline Layout gateup_layout(int H, int G, int B, int fmt, int NT) {
    Layout L;
    const int nblk = H / 64, ng = H / G;
    L.planes = 0;
    L.meta = align16(static_cast<size_t>(2) * B * nblk * 128);
    const size_t meta_bytes = fmt == DPA_FMT_UNIFORM ? static_cast<size_t>(2) * 16 * ng * 4
                                                     : static_cast<size_t>(2) * B * 16 * ng * 2;
    L.dig = align16(L.meta + meta_bytes);
    L.dig_stride = H + kDigPad;
    const size_t sl = static_cast<size_t>(2 * NT);   // token slots of one pass
    L.xe = align16(L.dig + sl * 3 * L.dig_stride);
    L.xs = align16(L.xe + sl * ng * 4);
    L.red = align16(L.xs + sl * ng * 4);
    L.total = align16(L.red + static_cast<size_t>(kWarps) * NT * 2 * 2 * 16 * 4);
    return L;
}

// down: planes [B][4][nblk][32], meta, digits [2NT][3][I+pad], exps/sums [2NT][ng]
__host__ __device__ inline Layout down_layout(int I, int G, int B, int fmt, int NT) {
    Layout L;
    const int nblk = I / 64, ng = I / G;
    L.planes = 0;
    L.meta = align16(static_cast<size_t>(B) * 4 * nblk * 128);
    const size_t meta_bytes = fmt == DPA_FMT_UNIFORM ? static_cast<size_t>(64) * ng * 4
                                                     : static_cast<size_t>(B) * 64 * ng * 2;
    L.dig = align16(L.meta + meta_bytes);
    L.dig_stride = I + kDigPad;
    const size_t sl = static_cast<size_t>(2 * NT);   // pair slots of one pass
    L.xe = align16(L.dig + sl * 3 * L.dig_stride);
    L.xs = align16(L.xe + sl * ng * 4);
    L.red = align16(L.xs + sl * ng * 4);
    L.total = align16(L.red + static_cast<size_t>(2) * 4 * NT * 2 * 16 * 4);
    return L;
}

// ---------------------------------------------------------------------------------------
// gate + up projections, SwiGLU epilogue -> h[pos][I]
// ---------------------------------------------------------------------------------------
template <int FMT, int B, int NT>
__global__ void __launch_bounds__(kThreads, NT > 1 ? 2 : 0) gateup_kernel(GemvArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int H = a.H, I = a.I, G = a.G;
    const int nblk = H >> 6, ng = H / G, bpg = G >> 6;
    const int tiles_per_expert = I >> 4;
    const Layout Ly = gateup_layout(H, G, B, FMT, NT);
    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem + Ly.planes);
    unsigned char* s_meta = smem + Ly.meta;
    int8_t* s_dig = reinterpret_cast<int8_t*>(smem + Ly.dig);
    int* s_xe = reinterpret_cast<int*>(smem + Ly.xe);
    int* s_xs = reinterpret_cast<int*>(smem + Ly.xs);
    float* s_red = reinterpret_cast<float*>(smem + Ly.red);
    __shared__ uint64_t s_bar, s_bard;   // planes and scales; the pass's digits
    __shared__ int s_flag;
    __shared__ int4 s_tile[NT];
    __shared__ int s_nt;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tq = lane & 3;
    if (threadIdx.x == 0) {
        mbar_init(&s_bar, 1);
        mbar_init(&s_bard, 1);
        fence_barrier_init();
    }
    const int dstride = Ly.dig_stride;
    // A single token (P == K) sits in the first half of every tile. Its digits were written by
    // the router two launches back, which completed before the previous launch passed its own
    // dependency wait, so they are staged before this kernel's wait (L2 reads).
    const bool single = NT == 1 && a.P == a.K;
    if (single) {
        const int chunks = (3 * H) >> 4;
        for (int c = threadIdx.x; c < 2 * chunks; c += kThreads) {
            const int slot = c / chunks, cc = c - slot * chunks;
            const uint4 v = slot == 0 ? __ldcg(reinterpret_cast<const uint4*>(a.xdig) + cc) : make_uint4(0u, 0u, 0u, 0u);
            const int d_ = (16 * cc) / H, col = 16 * cc - d_ * H;
            *reinterpret_cast<uint4*>(s_dig + (slot * 3 + d_) * dstride + col) = v;
        }
        for (int i = threadIdx.x; i < 2 * ng; i += kThreads) {
            s_xe[i] = i < ng ? __ldcg(a.xexp + i) : 0;
            s_xs[i] = i < ng ? __ldcg(a.xsum + i) : 0;
        }
    }
    pdl_wait();   // work lists and activations come from the previous kernels
    pdl_trigger();   // the down kernel may become resident and fetch its first planes
    const int n_items = static_cast<int>(a.hdr->n_active) * tiles_per_expert;
    __syncthreads();
    uint32_t phase = 0, phase_d = 0;
    const bool copy_es = (ng & 3) == 0;   // exponent and sum rows are whole 16-byte units
    const int g0 = (warp * ng) / kWarps, g1 = ((warp + 1) * ng) / kWarps;   // this warp's groups
    const int dig = gid & 3, half = gid >> 2, my_half = tq >> 1;

    // the first item's descriptor is loaded together with the active count (the index is in
    // bounds for every launched CTA; its contents are used only if the item exists)
    int4 desc = a.exp_desc[2 * (blockIdx.x / tiles_per_expert)];
    int4 tile0 = a.exp_desc[2 * (blockIdx.x / tiles_per_expert) + 1];
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (item != blockIdx.x) {
            desc = a.exp_desc[2 * (item / tiles_per_expert)];
            tile0 = a.exp_desc[2 * (item / tiles_per_expert) + 1];
        }
        const int e = desc.x, kmax_e = desc.y, ntiles = desc.z, toff = desc.w;
        const int rt = item % tiles_per_expert;
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
        bool waited = false;
        for (int pass0 = 0; pass0 < ntiles; pass0 += NT) {
            if (NT == 1) {
                if (threadIdx.x == 0) s_tile[0] = pass0 == 0 ? tile0 : a.tiles[toff + pass0];
            } else if (threadIdx.x < NT) {
                const int i = threadIdx.x;
                s_tile[i] = pass0 + i < ntiles ? a.tiles[toff + pass0 + i] : make_int4(0, -1, -1, -1);
            }
            if (threadIdx.x == 0) s_nt = min(NT, ntiles - pass0);
            __syncthreads();
            const int nt = s_nt;
            // stage the digits, exponents and sums of the pass's tokens: loads issued first
            // (one- and two-token passes), or bulk copies (multi-token passes)
            if (NT == 1 && !single) {
                const int chunks = (3 * H) >> 4;
                for (int i0 = threadIdx.x; i0 < 2 * NT * chunks; i0 += 4 * kThreads) {
                    uint4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + u * kThreads;
                        v[u] = make_uint4(0u, 0u, 0u, 0u);
                        if (i < 2 * NT * chunks) {
                            const int slot = i / chunks, c = i - slot * chunks;
                            const int tok = tile_tok(s_tile[slot >> 1], slot & 1);
                            if (tok >= 0)
                                v[u] = *reinterpret_cast<const uint4*>(a.xdig + static_cast<size_t>(tok) * 3 * H + 16 * c);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + u * kThreads;
                        if (i < 2 * NT * chunks) {
                            const int slot = i / chunks, c = i - slot * chunks;
                            const int d_ = (16 * c) / H, col = 16 * c - d_ * H;
                            *reinterpret_cast<uint4*>(s_dig + (slot * 3 + d_) * dstride + col) = v[u];
                        }
                    }
                }
                for (int i = threadIdx.x; i < 2 * NT * ng; i += kThreads) {
                    const int slot = i / ng, g = i - slot * ng;
                    const int tok = tile_tok(s_tile[slot >> 1], slot & 1);
                    s_xe[i] = tok >= 0 ? a.xexp[tok * ng + g] : 0;
                    s_xs[i] = tok >= 0 ? a.xsum[tok * ng + g] : 0;
                }
            }
            if constexpr (NT > 1) {
                if (warp == 0)
                    issue_digit_copies<NT>(lane < 2 * NT ? tile_tok(s_tile[lane >> 1], lane & 1) : -1, a.xdig, a.xexp,
                                           a.xsum, H, ng, copy_es, s_dig, dstride, s_xe, s_xs, &s_bard);
                if (!copy_es) {
                    for (int i = threadIdx.x; i < 2 * NT * ng; i += kThreads) {
                        const int slot = i / ng, g = i - slot * ng;
                        const int tok = tile_tok(s_tile[slot >> 1], slot & 1);
                        s_xe[i] = tok >= 0 ? a.xexp[tok * ng + g] : 0;
                        s_xs[i] = tok >= 0 ? a.xsum[tok * ng + g] : 0;
                    }
                }
                const bool okd = cta_wait_copies(&s_bard, phase_d, a.hdr, 104, &s_flag);
                phase_d ^= 1;
                if (!okd) return;
            }
            if (!waited) {
                waited = true;
                const bool ok = cta_wait_copies(&s_bar, phase, a.hdr, 100, &s_flag);
                phase ^= 1;
                if (!ok) return;
            } else {
                __syncthreads();
            }

            float acc[NT][2][2];
#pragma unroll
            for (int i = 0; i < NT; ++i)
#pragma unroll
                for (int m = 0; m < 2; ++m) acc[i][m][0] = acc[i][m][1] = 0.f;
            const int8_t* brow[NT];
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                const int slot = 2 * i + half;
                const int tk_ = tile_tok(s_tile[i], half);
                brow[i] = (i < nt && dig < 3 && tk_ >= 0) ? s_dig + (slot * 3 + dig) * dstride : nullptr;
            }
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
                        const uint32_t* pg = s_planes + static_cast<size_t>(b) * 32 + lane;   // gate, plane 0
                        const uint32_t* pu = pg + static_cast<size_t>(B) * nblk * 32;         // up, plane 0
                        const int ps = nblk * 32;                                             // plane stride
                        uint32_t R[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
                        int cur = 0;
                        uint32_t Alo[2][4], Ahi[2][4];
#pragma unroll
                        for (int i = 0; i < NT; ++i) {
                            if (i < nt) {
                                const int ki = s_tile[i].x;
                                if (ki > cur) {
                                    add_planes<B>(R[0], pg, ps, cur, ki);
                                    add_planes<B>(R[1], pu, ps, cur, ki);
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
                                if (brow[i]) load_b(brow[i], b, tq, b0L, b1L, b0H, b1H);
#pragma unroll
                                for (int m = 0; m < 2; ++m) {
                                    mma_u8s8(C[i][m][0], Alo[m][0], Alo[m][1], Alo[m][2], Alo[m][3], b0L, b1L);
                                    mma_u8s8(C[i][m][1], Ahi[m][0], Ahi[m][1], Ahi[m][2], Ahi[m][3], b0H, b1H);
                                }
                            }
                        }
                    }
                    const uint32_t* meta_u = reinterpret_cast<const uint32_t*>(s_meta);
#pragma unroll
                    for (int i = 0; i < NT; ++i) {
                        if (i < nt) {
                            const int slot = 2 * i + my_half;
                            const int ki = s_tile[i].x;
                            const float ck = 0.5f * static_cast<float>((1 << (B - ki)) - 1);
                            int Eg, SX;
                            Eg = s_xe[slot * ng + g];
                            SX = s_xs[slot * ng + g];
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
                                    uint32_t R[4] = {0u, 0u, 0u, 0u};
                                    add_plane<0>(R, s_planes[(static_cast<size_t>(m * B + p) * nblk + b) * 32 + lane]);
#pragma unroll
                                    for (int r = 0; r < 4; ++r) {
                                        Alo[m][r] = R[r] & 0x0F0F0F0Fu;
                                        Ahi[m][r] = R[r] & 0xF0F0F0F0u;
                                    }
                                }
#pragma unroll
                                for (int i = 0; i < NT; ++i) {
                                    if (i < nt && s_tile[i].x > p) {
                                        uint32_t b0L = 0, b1L = 0, b0H = 0, b1H = 0;
                                        if (brow[i]) load_b(brow[i], b, tq, b0L, b1L, b0H, b1H);
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
                                if (i < nt && s_tile[i].x > p) {
                                    const int slot = 2 * i + my_half;
                                    int Eg, SX;
                            Eg = s_xe[slot * ng + g];
                            SX = s_xs[slot * ng + g];
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
                            s_red[((((warp * NT + i) * 2 + m) * 2 + my_half) * 16) + gid + 8 * rr] = acc[i][m][rr];
            }
            __syncthreads();
            for (int q = threadIdx.x; q < NT * 32; q += kThreads) {
                const int i = q >> 5, tk = (q >> 4) & 1, row = q & 15;
                if (i < nt) {
                    const int pos = tk ? s_tile[i].z : s_tile[i].y;
                    if (pos >= 0) {
                        float ag = 0.f, au = 0.f;
#pragma unroll
                        for (int w = 0; w < kWarps; ++w) {
                            ag += s_red[((((w * NT + i) * 2 + 0) * 2 + tk) * 16) + row];
                            au += s_red[((((w * NT + i) * 2 + 1) * 2 + tk) * 16) + row];
                        }
                        a.h[static_cast<size_t>(pos) * I + rt * 16 + row] = ag / (1.f + expf(-ag)) * au;
                    }
                }
            }
            __syncthreads();
        }
        if (!waited) {   // no tiles (cannot happen for an active expert): keep the phase in step
            const bool ok = cta_wait_copies(&s_bar, phase, a.hdr, 102, &s_flag);
            phase ^= 1;
            if (!ok) return;
        }
    }
}

// ---------------------------------------------------------------------------------------
// down projection: out_pair[pos][H] = W_down^(k) h[pos]
// ---------------------------------------------------------------------------------------
template <int FMT, int B, int NT>
__global__ void __launch_bounds__(kThreads, NT > 1 ? 2 : 0) down_kernel(GemvArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int H = a.H, I = a.I, G = a.G;
    const int nblk = I >> 6, ng = I / G, bpg = G >> 6;
    const int tiles_per_expert = H >> 6;   // 64-row items: 4 row tiles x 2 K halves = 8 warps
    const Layout Ly = down_layout(I, G, B, FMT, NT);
    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem + Ly.planes);
    unsigned char* s_meta = smem + Ly.meta;
    int8_t* s_dig = reinterpret_cast<int8_t*>(smem + Ly.dig);
    int* s_xe = reinterpret_cast<int*>(smem + Ly.xe);
    int* s_xs = reinterpret_cast<int*>(smem + Ly.xs);
    float* s_red = reinterpret_cast<float*>(smem + Ly.red);   // [2 halves][4 tiles][NT][2][16]
    __shared__ uint64_t s_bar, s_bard;   // planes and scales; the pass's h digits (multi-token)
    __shared__ int s_flag;
    __shared__ int4 s_tile[NT];
    __shared__ int s_nt;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tq = lane & 3;
    if (threadIdx.x == 0) {
        mbar_init(&s_bar, 1);
        mbar_init(&s_bard, 1);
        fence_barrier_init();
    }
    // The work lists come from the allocation, which completed before the gate/up kernel (this
    // kernel's predecessor) passed its own dependency wait, and the planes are static: the first
    // item's descriptor is read (from L2) and its plane copies issued before this kernel's wait.
    const int n_items = static_cast<int>(__ldcg(&a.hdr->n_active)) * tiles_per_expert;
    int4 desc = __ldcg(a.exp_desc + 2 * (blockIdx.x / tiles_per_expert));
    int4 tile0 = __ldcg(a.exp_desc + 2 * (blockIdx.x / tiles_per_expert) + 1);
    auto issue_planes = [&](const int4& d, int rt) {   // thread 0: the item's planes and scales
        const int e = d.x, kmax_e = d.y;
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
    };
    if (threadIdx.x == 0 && static_cast<int>(blockIdx.x) < n_items) issue_planes(desc, blockIdx.x % tiles_per_expert);
    pdl_wait();   // h and its digits come from the previous kernel
    __syncthreads();
    uint32_t phase = 0, phase_d = 0;
    const int dig = gid & 3, half = gid >> 2, my_half = tq >> 1;
    const int dstride = Ly.dig_stride;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (item != blockIdx.x) {
            desc = a.exp_desc[2 * (item / tiles_per_expert)];
            tile0 = a.exp_desc[2 * (item / tiles_per_expert) + 1];
        }
        const int kmax_e = desc.y, ntiles = desc.z, toff = desc.w;
        const int rt = item % tiles_per_expert;
        if (threadIdx.x == 0 && item != static_cast<int>(blockIdx.x)) issue_planes(desc, rt);
        bool waited = false;
        for (int pass0 = 0; pass0 < ntiles; pass0 += NT) {
            if (NT == 1) {
                if (threadIdx.x == 0) s_tile[0] = pass0 == 0 ? tile0 : a.tiles[toff + pass0];
            } else if (threadIdx.x < NT) {
                const int i = threadIdx.x;
                s_tile[i] = pass0 + i < ntiles ? a.tiles[toff + pass0 + i] : make_int4(0, -1, -1, -1);
            }
            if (threadIdx.x == 0) s_nt = min(NT, ntiles - pass0);
            __syncthreads();
            const int nt = s_nt;
            // fixed-point digits of the pass's h rows: one warp per (slot, group); a lane holds
            // 4 consecutive values per 128-column chunk, all loaded before use
            for (int task = warp; NT == 1 && task < 2 * NT * ng; task += kWarps) {
                const int slot = task / ng, g = task - slot * ng;
                const int4 t = s_tile[slot >> 1];
                const int pos = (slot & 1) ? t.z : t.y;
                if (pos < 0) continue;
                const float* hrow = a.h + static_cast<size_t>(pos) * I + g * G;
                float4 hv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = 128 * u + 4 * lane;
                    hv[u] = j < G ? *reinterpret_cast<const float4*>(hrow + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                float mx = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(hv[u].x), fabsf(hv[u].y)), fmaxf(fabsf(hv[u].z), fabsf(hv[u].w))));
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const int Eg = group_exponent(mx);
                int sum = 0;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = 128 * u + 4 * lane;
                    if (j < G) {
                        const float vv[4] = {hv[u].x, hv[u].y, hv[u].z, hv[u].w};
                        uint32_t p0 = 0, p1 = 0, p2 = 0;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int X = to_fixed(vv[q], Eg);
                            sum += X;
                            int8_t d0, d1, d2;
                            split_digits(X, d0, d1, d2);
                            p0 |= static_cast<uint32_t>(static_cast<uint8_t>(d0)) << (8 * q);
                            p1 |= static_cast<uint32_t>(static_cast<uint8_t>(d1)) << (8 * q);
                            p2 |= static_cast<uint32_t>(static_cast<uint8_t>(d2)) << (8 * q);
                        }
                        int8_t* dst = s_dig + (slot * 3) * dstride + g * G + j;
                        *reinterpret_cast<uint32_t*>(dst) = p0;
                        *reinterpret_cast<uint32_t*>(dst + dstride) = p1;
                        *reinterpret_cast<uint32_t*>(dst + 2 * dstride) = p2;
                    }
                }
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) { s_xe[slot * ng + g] = Eg; s_xs[slot * ng + g] = sum; }
            }
            if constexpr (NT > 1) {   // digits of every h row were written by hdigits_kernel
                if (warp == 0)
                    issue_digit_copies<NT>(lane < 2 * NT ? ((lane & 1) ? s_tile[lane >> 1].z : s_tile[lane >> 1].y) : -1,
                                           a.hdig, a.hexp, a.hsum, I, ng, (ng & 3) == 0, s_dig, dstride, s_xe, s_xs,
                                           &s_bard);
                if ((ng & 3) != 0) {
                    for (int i = threadIdx.x; i < 2 * NT * ng; i += kThreads) {
                        const int slot = i / ng, g = i - slot * ng;
                        const int4 t = s_tile[slot >> 1];
                        const int pos = (slot & 1) ? t.z : t.y;
                        s_xe[i] = pos >= 0 ? a.hexp[pos * ng + g] : 0;
                        s_xs[i] = pos >= 0 ? a.hsum[pos * ng + g] : 0;
                    }
                }
                const bool okd = cta_wait_copies(&s_bard, phase_d, a.hdr, 204, &s_flag);
                phase_d ^= 1;
                if (!okd) return;
            }
            if (!waited) {
                waited = true;
                const bool ok = cta_wait_copies(&s_bar, phase, a.hdr, 200, &s_flag);
                phase ^= 1;
                if (!ok) return;
            } else {
                __syncthreads();
            }

            float acc[NT][2];
#pragma unroll
            for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = 0.f;
            const int8_t* brow[NT];
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                const int slot = 2 * i + half;
                const int4 t = s_tile[i];
                const int pos = half ? t.z : t.y;
                brow[i] = (i < nt && dig < 3 && pos >= 0) ? s_dig + (slot * 3 + dig) * dstride : nullptr;
            }
            const int rtile = warp & 3, khalf = warp >> 2;   // row tile of 4, half of the groups
            const uint32_t* wplanes = s_planes + static_cast<size_t>(rtile) * nblk * 32;
            const int gbeg = (khalf * ng) / 2, gend = ((khalf + 1) * ng) / 2;
            for (int g = gbeg; g < gend; ++g) {
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
                        const uint32_t* pw = wplanes + static_cast<size_t>(b) * 32 + lane;   // plane 0
                        const int ps = 4 * nblk * 32;                                        // plane stride
                        uint32_t R[4] = {0u, 0u, 0u, 0u};
                        int cur = 0;
                        uint32_t Alo[4], Ahi[4];
#pragma unroll
                        for (int i = 0; i < NT; ++i) {
                            if (i < nt) {
                                const int ki = s_tile[i].x;
                                if (ki > cur) {
                                    add_planes<B>(R, pw, ps, cur, ki);
                                    cur = ki;
#pragma unroll
                                    for (int r = 0; r < 4; ++r) {
                                        Alo[r] = R[r] & 0x0F0F0F0Fu;
                                        Ahi[r] = R[r] & 0xF0F0F0F0u;
                                    }
                                }
                                uint32_t b0L = 0, b1L = 0, b0H = 0, b1H = 0;
                                if (brow[i]) load_b(brow[i], b, tq, b0L, b1L, b0H, b1H);
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
                            const int ki = s_tile[i].x;
                            const float ck = 0.5f * static_cast<float>((1 << (B - ki)) - 1);
                            int Eg, SX;
                            Eg = s_xe[slot * ng + g];
                            SX = s_xs[slot * ng + g];
                            const float sc2 = pow2f(Eg - 22);
#pragma unroll
                            for (int rr = 0; rr < 2; ++rr) {
                                float v = digit_value(C[i][0][2 * rr], C[i][1][2 * rr], C[i][0][2 * rr + 1], C[i][1][2 * rr + 1], tq);
                                v += __shfl_xor_sync(0xffffffffu, v, 1);
                                const int row = rtile * 16 + gid + 8 * rr;
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
                                uint32_t R[4] = {0u, 0u, 0u, 0u};
                                add_plane<0>(R, wplanes[(static_cast<size_t>(p) * 4 * nblk + b) * 32 + lane]);
                                uint32_t Alo[4], Ahi[4];
#pragma unroll
                                for (int r = 0; r < 4; ++r) {
                                    Alo[r] = R[r] & 0x0F0F0F0Fu;
                                    Ahi[r] = R[r] & 0xF0F0F0F0u;
                                }
#pragma unroll
                                for (int i = 0; i < NT; ++i) {
                                    if (i < nt && s_tile[i].x > p) {
                                        uint32_t b0L = 0, b1L = 0, b0H = 0, b1H = 0;
                                        if (brow[i]) load_b(brow[i], b, tq, b0L, b1L, b0H, b1H);
                                        mma_u8s8(C[i][0], Alo[0], Alo[1], Alo[2], Alo[3], b0L, b1L);
                                        mma_u8s8(C[i][1], Ahi[0], Ahi[1], Ahi[2], Ahi[3], b0H, b1H);
                                    }
                                }
                            }
#pragma unroll
                            for (int i = 0; i < NT; ++i) {
                                if (i < nt && s_tile[i].x > p) {
                                    const int slot = 2 * i + my_half;
                                    int Eg, SX;
                            Eg = s_xe[slot * ng + g];
                            SX = s_xs[slot * ng + g];
                                    const float sc2 = pow2f(Eg - 22);
#pragma unroll
                                    for (int rr = 0; rr < 2; ++rr) {
                                        float v = digit_value(C[i][0][2 * rr], C[i][1][2 * rr], C[i][0][2 * rr + 1],
                                                              C[i][1][2 * rr + 1], tq);
                                        v += __shfl_xor_sync(0xffffffffu, v, 1);
                                        const int row = rtile * 16 + gid + 8 * rr;
                                        const float al = __half2float(meta_h[(p * 64 + row) * ng + g]);
                                        acc[i][rr] = fmaf(al * sc2, fmaf(2.f, v, -static_cast<float>(SX)), acc[i][rr]);
                                    }
                                }
                            }
                        }
                    }
                }
            }
            // the two K halves meet in shared memory (fixed order), then one store per output
            if ((tq & 1) == 0) {
#pragma unroll
                for (int i = 0; i < NT; ++i)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr)
                        s_red[(((khalf * 4 + rtile) * NT + i) * 2 + my_half) * 16 + gid + 8 * rr] = acc[i][rr];
            }
            __syncthreads();
            for (int q = threadIdx.x; q < 4 * NT * 32; q += kThreads) {
                const int row = q & 15, tk = (q >> 4) & 1, i = (q >> 5) % NT, tl = q / (32 * NT);
                if (i < nt) {
                    const int pos = tk ? s_tile[i].z : s_tile[i].y;
                    if (pos >= 0) {
                        const float v = s_red[(((0 * 4 + tl) * NT + i) * 2 + tk) * 16 + row] +
                                        s_red[(((1 * 4 + tl) * NT + i) * 2 + tk) * 16 + row];
                        a.out_pair[static_cast<size_t>(pos) * H + rt * 64 + tl * 16 + row] = v;
                    }
                }
            }
            __syncthreads();
        }
        if (!waited) {
            const bool ok = cta_wait_copies(&s_bar, phase, a.hdr, 202, &s_flag);
            phase ^= 1;
            if (!ok) return;
        }
    }
}

// Fixed-point digits of every pair's SwiGLU row h[pos] (for the multi-token down kernel):
// one warp per (position, group), the same arithmetic as the staged per-CTA digits.
__global__ void __launch_bounds__(256) hdigits_kernel(GemvArgs a) {
    pdl_wait();
    const int I = a.I, G = a.G, ng = I / G;
    const int task = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (task >= a.P * ng) return;
    const int pos = task / ng, g = task - pos * ng;
    const float* hrow = a.h + static_cast<size_t>(pos) * I + g * G;
    float4 hv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int j = 128 * u + 4 * lane;
        hv[u] = j < G ? *reinterpret_cast<const float4*>(hrow + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mx = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u)
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(hv[u].x), fabsf(hv[u].y)), fmaxf(fabsf(hv[u].z), fabsf(hv[u].w))));
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const int Eg = group_exponent(mx);
    int sum = 0;
    int8_t* drow = a.hdig + static_cast<size_t>(pos) * 3 * I + g * G;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int j = 128 * u + 4 * lane;
        if (j < G) {
            const float vv[4] = {hv[u].x, hv[u].y, hv[u].z, hv[u].w};
            uint32_t p0 = 0, p1 = 0, p2 = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int X = to_fixed(vv[q], Eg);
                sum += X;
                int8_t d0, d1, d2;
                split_digits(X, d0, d1, d2);
                p0 |= static_cast<uint32_t>(static_cast<uint8_t>(d0)) << (8 * q);
                p1 |= static_cast<uint32_t>(static_cast<uint8_t>(d1)) << (8 * q);
                p2 |= static_cast<uint32_t>(static_cast<uint8_t>(d2)) << (8 * q);
            }
            *reinterpret_cast<uint32_t*>(drow + j) = p0;
            *reinterpret_cast<uint32_t*>(drow + I + j) = p1;
            *reinterpret_cast<uint32_t*>(drow + 2 * I + j) = p2;
        }
    }
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
        a.hexp[pos * ng + g] = Eg;
        a.hsum[pos * ng + g] = sum;
    }
}

template <int FMT, int NT>
void* pick_gateup(int B) {
    switch (B) {
        case 1: return reinterpret_cast<void*>(gateup_kernel<FMT, 1, NT>);
        case 2: return reinterpret_cast<void*>(gateup_kernel<FMT, 2, NT>);
        case 3: return reinterpret_cast<void*>(gateup_kernel<FMT, 3, NT>);
        default: return reinterpret_cast<void*>(gateup_kernel<FMT, 4, NT>);
    }
}
template <int FMT, int NT>
void* pick_down(int B) {
    switch (B) {
        case 1: return reinterpret_cast<void*>(down_kernel<FMT, 1, NT>);
        case 2: return reinterpret_cast<void*>(down_kernel<FMT, 2, NT>);
        case 3: return reinterpret_cast<void*>(down_kernel<FMT, 3, NT>);
        default: return reinterpret_cast<void*>(down_kernel<FMT, 4, NT>);
    }
}

// tiles per pass: 4 when experts may hold more than two tokens and the multi-token staging of
// both kernels fits in shared memory, else 1
int pick_nt(const GemvArgs& a) {
    if (a.max_tokens_per_expert <= 2) return 1;
    const bool fits = gateup_layout(a.H, a.G, a.B, a.fmt, 4).total <= kGemvMaxSmem &&
                      down_layout(a.I, a.G, a.B, a.fmt, 4).total <= kGemvMaxSmem;
    return fits ? 4 : 1;
}

cudaError_t launch_generic(void* fn, size_t smem, int items, int num_sms, const GemvArgs& a, cudaStream_t stream) {
    if (items <= 0) return cudaSuccess;
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    const int grid = items < num_sms * per_sm ? items : num_sms * per_sm;
    GemvArgs copy = a;
    void* args[] = {&copy};
    return launch_pdl_raw(fn, dim3(grid), dim3(kThreads), smem, stream, args);
}

}  // namespace

size_t gateup_smem_bytes(const GemvArgs& a) { return gateup_layout(a.H, a.G, a.B, a.fmt, 1).total; }
size_t down_smem_bytes(const GemvArgs& a) { return down_layout(a.I, a.G, a.B, a.fmt, 1).total; }

cudaError_t launch_gateup(const GemvArgs& a, cudaStream_t stream, int num_sms) {
    const int nt = pick_nt(a);
    void* fn;
    if (a.fmt == DPA_FMT_UNIFORM) fn = nt == 1 ? pick_gateup<DPA_FMT_UNIFORM, 1>(a.B) : pick_gateup<DPA_FMT_UNIFORM, 4>(a.B);
    else fn = nt == 1 ? pick_gateup<DPA_FMT_BCQ, 1>(a.B) : pick_gateup<DPA_FMT_BCQ, 4>(a.B);
    return launch_generic(fn, gateup_layout(a.H, a.G, a.B, a.fmt, nt).total, a.max_items * (a.I >> 4), num_sms, a,
                          stream);
}

cudaError_t launch_down(const GemvArgs& a, cudaStream_t stream, int num_sms) {
    const int nt = pick_nt(a);
    if (nt > 1) {   // digits of every h row once, for the multi-token down kernel
        const int tasks = a.P * (a.I / a.G);
        GemvArgs copy = a;
        void* args[] = {&copy};
        cudaError_t err = launch_pdl_raw(reinterpret_cast<const void*>(hdigits_kernel), dim3((tasks + 7) / 8), dim3(256),
                                         0, stream, args);
        if (err != cudaSuccess) return err;
    }
    void* fn;
    if (a.fmt == DPA_FMT_UNIFORM) fn = nt == 1 ? pick_down<DPA_FMT_UNIFORM, 1>(a.B) : pick_down<DPA_FMT_UNIFORM, 4>(a.B);
    else fn = nt == 1 ? pick_down<DPA_FMT_BCQ, 1>(a.B) : pick_down<DPA_FMT_BCQ, 4>(a.B);
    return launch_generic(fn, down_layout(a.I, a.G, a.B, a.fmt, nt).total, a.max_items * (a.H >> 6), num_sms, a,
                          stream);
}

}  // namespace dpa
