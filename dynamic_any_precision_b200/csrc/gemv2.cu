// Pipelined variable-plane expert GEMV for decode-sized batches (the hot path).
//
// Each routed pair reads only the first k planes of its expert's matrices (DPA-MoE, Abstract:
// chunks that decode by prefix; DuoRate, Abstract: a weight stream readable by prefix; MatMoE,
// review "Core Contribution": bitplane storage and floor-and-compensation). For uniform codes
// with B planes and a pair reading k of them, per scale group g of a row:
//   sum_j s_g (q_hat_j - z_g) x_j = s_g [ sum_j qtrunc_j x_j + (c_k - z_g) sum_j x_j ],
//   qtrunc_j = the code with its B-k low bits cleared,  c_k = (2^(B-k) - 1) / 2.
// For binary-coded planes (b = +-1, per-plane scale alpha_p) it is sum_{p<k} alpha_p (2 S_p - X),
// S_p = the sum of x over the plane's +1 bits and X = the sum of x over the group.
//
// Activations (x per token, or the SwiGLU output h per pair) arrive as fixed point per scale
// group: X_j = rint(v_j 2^(14-E)) with |v| < 2^E, split into two int8 digits d0 + 256 d1, the
// s8 operand of a u8 x s8 mma.sync (m16n8k32, exact int32 accumulation); an n8 column tile holds
// four tokens x two digits. The weight operand is the u8 code: the plane words of a lane are
// gathered into nibbles (one register of eight 4-bit codes per nibble position rho), split into
// the low and high nibbles of each byte, and masked to the k planes a token tile reads.
//
// Work: items are (token group, row block). A token group is up to NTILE tiles of up to four
// pairs of one expert, each tile of one plane count k (tiles ascending in k). One CTA per SM,
// persistent over its items:
//   - warp 16 (producer) streams each item's columns in chunks into a ring of stages with bulk
//     copies (no multicast): for every matrix and plane p < kmax of the group and every row
//     tile, the chunk's plane words; the chunk's digit rows of the group's tokens; with the
//     item's first chunk also its scales and the tokens' group exponents and sums;
//   - warps 0-15 (consumers) take row tile rt and column slice cs of every chunk; they wait for
//     a stage's full barrier, compute, and release it through the stage's empty barrier;
//   - at the end of an item the column slices of a row tile are summed in a fixed order and the
//     epilogue (SwiGLU for gate/up, the per-pair output for down) is written.
// Every wait is bounded (globaltimer); on a timeout the kernel records DPA_ERR_DEVICE_TIMEOUT,
// sets a CTA-wide abort flag that ends every other wait, and the producer waits for the copies
// it issued before the CTA exits.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kCW = 8;                        // consumer warps
constexpr int kVThreads = (kCW + 1) * 32;     // + the producer warp
constexpr int kMaxStages = 8;                 // ring depth: as many stages as shared memory holds
constexpr int kMaxB = 4;
constexpr int kDigPad = 64;                   // bytes of padding per staged digit row (banks)

template <int NRT>
struct Geo {
    static constexpr int CS = kCW / NRT;      // column slices per chunk
    static constexpr int CWS = 128;           // columns per slice (two 64-column blocks)
    static constexpr int CK = CS * CWS;       // columns per chunk
    static constexpr int RB = 16 * NRT;       // rows per item
};

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~static_cast<size_t>(15); }
__host__ __device__ inline size_t al128(size_t v) { return (v + 127) & ~static_cast<size_t>(127); }

struct VLayout {                             // byte offsets in dynamic shared memory (< 227 KB)
    uint32_t stage, st_dig, dig_stride;       // per stage: planes at 0, digits at st_dig
    uint32_t slot, sl_exp, sl_sum, sl_tab;    // per item slot: meta at 0, then exps, sums, table
    uint32_t red, red_per;                    // reduction buffer (NRT x (CS-1) warps)
    uint32_t total;
    int nst;                                  // stages in the ring
    int ngp;                                  // exps/sums row stride (ints)
};

template <int NRT, int NTILE, int NMAT>
__host__ __device__ inline VLayout vlayout(int K, int G, int fmt, int B) {
    using Gm = Geo<NRT>;
    VLayout L;
    const size_t ng = K / G;
    L.ngp = static_cast<int>((ng + 3) & ~static_cast<size_t>(3));
    const size_t dig_stride = Gm::CK + kDigPad;
    const size_t planes = static_cast<size_t>(NMAT) * kMaxB * NRT * (Gm::CK / 64) * 128;
    const size_t stage = al128(planes + static_cast<size_t>(4 * NTILE) * 2 * dig_stride);
    const size_t meta = fmt == DPA_FMT_UNIFORM ? static_cast<size_t>(NMAT) * Gm::RB * ng * 4
                                               : static_cast<size_t>(NMAT) * B * Gm::RB * ng * 2;
    const size_t sl_exp = al16(meta);
    const size_t sl_sum = sl_exp + static_cast<size_t>(4 * NTILE) * L.ngp * 4;
    const size_t sl_tab = sl_sum + static_cast<size_t>(4 * NTILE) * L.ngp * 4;
    // table: {e, kmax, ntiles, rb}, NTILE x {k, n, 0, 0}, 4*NTILE digit rows, 4*NTILE output rows
    const size_t slot = al128(sl_tab + 16 + 16 * NTILE + 8 * 4 * NTILE);
    const size_t red_per = static_cast<size_t>(32) * NTILE * NMAT * 2 * 4;
    const size_t fixed = 2 * slot + static_cast<size_t>(NRT) * (Gm::CS - 1) * red_per;
    int nst = 2;   // at least double buffering; more while the ring fits beside the fixed parts
    while (nst < kMaxStages && fixed + (nst + 1) * stage <= kVpMaxSmem) ++nst;
    const size_t red = nst * stage + 2 * slot;
    size_t total = red + static_cast<size_t>(NRT) * (Gm::CS - 1) * red_per;
    if (total > 0xFFFFFFFFull) total = 0xFFFFFFFFull;   // rejected by the caller (too large)
    L.nst = nst;
    L.stage = static_cast<uint32_t>(stage);
    L.st_dig = static_cast<uint32_t>(planes);
    L.dig_stride = static_cast<uint32_t>(dig_stride);
    L.slot = static_cast<uint32_t>(slot);
    L.sl_exp = static_cast<uint32_t>(sl_exp);
    L.sl_sum = static_cast<uint32_t>(sl_sum);
    L.sl_tab = static_cast<uint32_t>(sl_tab);
    L.red = static_cast<uint32_t>(red);
    L.red_per = static_cast<uint32_t>(red_per);
    L.total = static_cast<uint32_t>(total);
    return L;
}

// waits that end on a bounded time or on the CTA's abort flag
__device__ __forceinline__ bool vwait(uint64_t* bar, uint32_t parity, volatile int* abort, WsHeader* hdr,
                                      uint32_t where) {
    return mbar_wait_abortable(bar, parity, abort, hdr, where);
}

// ---- nibble assembly (as in the plane layout of dpa.h: bit 4m + rho of a lane's word) ----
template <int RHO, int T>
__device__ __forceinline__ uint32_t nibs(uint32_t w) {
    uint32_t v;
    if constexpr (T >= RHO) v = w << (T - RHO);
    else v = w >> (RHO - T);
    return v & (0x11111111u << T);
}
template <int T>
__device__ __forceinline__ void add_plane(uint32_t (&R)[4], uint32_t w) {
    R[0] |= nibs<0, T>(w);
    R[1] |= nibs<1, T>(w);
    R[2] |= nibs<2, T>(w);
    R[3] |= nibs<3, T>(w);
}
// planes [0, kmax) of one lane's words (plane p at w[p]); code bit of plane p = B-1-p
template <int B>
__device__ __forceinline__ void assemble(uint32_t (&R)[4], const uint32_t (&w)[kMaxB], int kmax) {
    R[0] = R[1] = R[2] = R[3] = 0u;
    if constexpr (B >= 1) add_plane<B - 1>(R, w[0]);
    if constexpr (B >= 2) if (kmax > 1) add_plane<B - 2>(R, w[1]);
    if constexpr (B >= 3) if (kmax > 2) add_plane<B - 3>(R, w[2]);
    if constexpr (B >= 4) if (kmax > 3) add_plane<0>(R, w[3]);
}
// the codes of a k-plane read: the top k of B bits of every nibble, in the low nibble of a byte
__device__ __forceinline__ uint32_t level_mask(int B, int k) {
    const uint32_t nib = ((1u << k) - 1u) << (B - k);
    return 0x0F0F0F0Fu & (nib * 0x01010101u);
}

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

// ---- B operand: the lane's 16 digit bytes of one 64-column block (one 16-byte load) ----
__device__ __forceinline__ uint4 lds128(const unsigned char* p) { return *reinterpret_cast<const uint4*>(p); }

template <int NRT, int NTILE, int NMAT>
struct Item {
    int e, kmax, nt, rb;
    int tk[NTILE], tn[NTILE];
};

// ---------------------------------------------------------------------------------------
// consumer: one column slice of one chunk, uniform codes
// ---------------------------------------------------------------------------------------
template <int B, int NRT, int NTILE, int NMAT>
__device__ __forceinline__ void slice_uniform(const VpArgs& a, const VLayout& L, const unsigned char* st,
                                              const unsigned char* sl, const Item<NRT, NTILE, NMAT>& it, int col0,
                                              int rt, int cs, float (&acc)[NTILE][NMAT][2]) {
    using Gm = Geo<NRT>;
    const int lane = threadIdx.x & 31, gid = lane >> 2, tq = lane & 3;
    const int G = a.G, K = a.K, ng = K / G;
    const uint32_t* planes = reinterpret_cast<const uint32_t*>(st);
    const unsigned char* dig = st + L.st_dig;
    const int* sexp = reinterpret_cast<const int*>(sl + L.sl_exp);
    const int* ssum = reinterpret_cast<const int*>(sl + L.sl_sum);
    int C[NTILE][NMAT][4];
#pragma unroll
    for (int t = 0; t < NTILE; ++t)
#pragma unroll
        for (int m = 0; m < NMAT; ++m) C[t][m][0] = C[t][m][1] = C[t][m][2] = C[t][m][3] = 0;
    bool has_start = false;
#pragma unroll 1
    for (int blk = 0; blk < 2; ++blk) {
        const int cb = cs * 2 + blk;                     // block inside the chunk
        const int colb = col0 + cb * 64;                 // global column of the block
        if (colb >= K) break;
        if (colb % G == 0) has_start = true;
        // the B fragments of the tiles (shared by the matrices), then one matrix at a time
        uint4 bt[NTILE];
#pragma unroll
        for (int t = 0; t < NTILE; ++t)
            if (t < it.nt)
                bt[t] = lds128(dig + static_cast<size_t>((4 * t + (gid >> 1)) * 2 + (gid & 1)) * L.dig_stride +
                               cb * 64 + 16 * tq);
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            uint32_t w[kMaxB];
#pragma unroll
            for (int p = 0; p < kMaxB; ++p)
                w[p] = p < it.kmax ? planes[(((m * kMaxB + p) * NRT + rt) * (Gm::CK / 64) + cb) * 32 + lane] : 0u;
            uint32_t R[4], Rh[4];
            assemble<B>(R, w, it.kmax);
#pragma unroll
            for (int r = 0; r < 4; ++r) Rh[r] = R[r] >> 4;
            int level = -1;
            uint32_t Alo[4], Ahi[4];
#pragma unroll
            for (int t = 0; t < NTILE; ++t) {
                if (t < it.nt) {
                    if (it.tk[t] != level) {
                        level = it.tk[t];
                        const uint32_t mk = level_mask(B, level);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            Alo[r] = R[r] & mk;
                            Ahi[r] = Rh[r] & mk;
                        }
                    }
                    mma_u8s8(C[t][m], Alo[0], Alo[1], Alo[2], Alo[3], bt[t].x, bt[t].y);
                    mma_u8s8(C[t][m], Ahi[0], Ahi[1], Ahi[2], Ahi[3], bt[t].z, bt[t].w);
                }
            }
        }
        // a group portion ends at the slice end, at the end of the columns, or at a group boundary
        const bool end = blk == 1 || colb + 64 >= K || (colb + 64) % G == 0;
        if (end) {
            const int g = colb / G;
            const uint32_t* meta = reinterpret_cast<const uint32_t*>(sl);
            float s[NMAT][2], z[NMAT][2];
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const uint32_t sz = meta[(m * Gm::RB + rt * 16 + gid + 8 * rr) * ng + g];
                    s[m][rr] = __half2float(__ushort_as_half(static_cast<unsigned short>(sz & 0xFFFFu)));
                    z[m][rr] = __half2float(__ushort_as_half(static_cast<unsigned short>(sz >> 16)));
                }
#pragma unroll
            for (int t = 0; t < NTILE; ++t) {
                if (t < it.nt) {
                    const int j = 4 * t + tq;
                    const float f = pow2i(sexp[j * L.ngp + g] - 14);
                    const float sx = has_start ? static_cast<float>(ssum[j * L.ngp + g]) : 0.f;
                    const float ck = 0.5f * static_cast<float>((1 << (B - it.tk[t])) - 1);
#pragma unroll
                    for (int m = 0; m < NMAT; ++m)
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            float v = static_cast<float>(C[t][m][2 * rr] + 256 * C[t][m][2 * rr + 1]);
                            v = fmaf(ck - z[m][rr], sx, v);
                            acc[t][m][rr] = fmaf(s[m][rr] * f, v, acc[t][m][rr]);
                            C[t][m][2 * rr] = C[t][m][2 * rr + 1] = 0;
                        }
                }
            }
            has_start = false;
        }
    }
}

// ---------------------------------------------------------------------------------------
// consumer: one column slice of one chunk, binary-coded planes
// ---------------------------------------------------------------------------------------
template <int B, int NRT, int NTILE, int NMAT>
__device__ __forceinline__ void slice_bcq(const VpArgs& a, const VLayout& L, const unsigned char* st,
                                          const unsigned char* sl, const Item<NRT, NTILE, NMAT>& it, int col0, int rt,
                                          int cs, float (&acc)[NTILE][NMAT][2]) {
    using Gm = Geo<NRT>;
    const int lane = threadIdx.x & 31, gid = lane >> 2, tq = lane & 3;
    const int G = a.G, K = a.K, ng = K / G;
    const uint32_t* planes = reinterpret_cast<const uint32_t*>(st);
    const unsigned char* dig = st + L.st_dig;
    const int* sexp = reinterpret_cast<const int*>(sl + L.sl_exp);
    const int* ssum = reinterpret_cast<const int*>(sl + L.sl_sum);
    const __half* meta = reinterpret_cast<const __half*>(sl);
    // the slice's blocks in group portions: [b0, b1) of blocks 0..1
    int b0 = 0;
    while (b0 < 2) {
        const int colb0 = col0 + (cs * 2 + b0) * 64;
        if (colb0 >= K) break;
        int b1 = b0 + 1;
        if (b1 < 2 && (colb0 + 64) % G != 0 && colb0 + 64 < K) b1 = 2;
        const int g = colb0 / G;
        const bool has_start = colb0 % G == 0;
#pragma unroll
        for (int p = 0; p < B; ++p) {
            if (p < it.kmax) {
                int C[NTILE][NMAT][4];
#pragma unroll
                for (int t = 0; t < NTILE; ++t)
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) C[t][m][0] = C[t][m][1] = C[t][m][2] = C[t][m][3] = 0;
                for (int blk = b0; blk < b1; ++blk) {
                    const int cb = cs * 2 + blk;
                    uint32_t lo[NMAT][4], hi[NMAT][4];
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        const uint32_t w = planes[(((m * kMaxB + p) * NRT + rt) * (Gm::CK / 64) + cb) * 32 + lane];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            lo[m][r] = (w >> r) & 0x01010101u;
                            hi[m][r] = (w >> (r + 4)) & 0x01010101u;
                        }
                    }
#pragma unroll
                    for (int t = 0; t < NTILE; ++t) {
                        if (t < it.nt && it.tk[t] > p) {
                            const uint4 b = lds128(dig +
                                                   static_cast<size_t>((4 * t + (gid >> 1)) * 2 + (gid & 1)) * L.dig_stride +
                                                   cb * 64 + 16 * tq);
#pragma unroll
                            for (int m = 0; m < NMAT; ++m) {
                                mma_u8s8(C[t][m], lo[m][0], lo[m][1], lo[m][2], lo[m][3], b.x, b.y);
                                mma_u8s8(C[t][m], hi[m][0], hi[m][1], hi[m][2], hi[m][3], b.z, b.w);
                            }
                        }
                    }
                }
                float al[NMAT][2];
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr)
                        al[m][rr] = __half2float(meta[((m * it.kmax + p) * Gm::RB + rt * 16 + gid + 8 * rr) * ng + g]);
#pragma unroll
                for (int t = 0; t < NTILE; ++t) {
                    if (t < it.nt && it.tk[t] > p) {
                        const int j = 4 * t + tq;
                        const float f = pow2i(sexp[j * L.ngp + g] - 14);
                        const float sx = has_start ? static_cast<float>(ssum[j * L.ngp + g]) : 0.f;
#pragma unroll
                        for (int m = 0; m < NMAT; ++m)
#pragma unroll
                            for (int rr = 0; rr < 2; ++rr) {
                                const float v = static_cast<float>(C[t][m][2 * rr] + 256 * C[t][m][2 * rr + 1]);
                                acc[t][m][rr] = fmaf(al[m][rr] * f, fmaf(2.f, v, -sx), acc[t][m][rr]);
                            }
                    }
                }
            }
        }
        b0 = b1;
    }
}

template <int FMT, int NRT, int NTILE, int NMAT>
__device__ __forceinline__ void slice_dispatch(const VpArgs& a, const VLayout& L, const unsigned char* st,
                                               const unsigned char* sl, const Item<NRT, NTILE, NMAT>& it, int col0,
                                               int rt, int cs, float (&acc)[NTILE][NMAT][2]) {
    if constexpr (FMT == DPA_FMT_UNIFORM) {
        switch (a.B) {
            case 1: slice_uniform<1, NRT, NTILE, NMAT>(a, L, st, sl, it, col0, rt, cs, acc); break;
            case 2: slice_uniform<2, NRT, NTILE, NMAT>(a, L, st, sl, it, col0, rt, cs, acc); break;
            case 3: slice_uniform<3, NRT, NTILE, NMAT>(a, L, st, sl, it, col0, rt, cs, acc); break;
            default: slice_uniform<4, NRT, NTILE, NMAT>(a, L, st, sl, it, col0, rt, cs, acc); break;
        }
    } else {
        switch (a.B) {
            case 1: slice_bcq<1, NRT, NTILE, NMAT>(a, L, st, sl, it, col0, rt, cs, acc); break;
            case 2: slice_bcq<2, NRT, NTILE, NMAT>(a, L, st, sl, it, col0, rt, cs, acc); break;
            case 3: slice_bcq<3, NRT, NTILE, NMAT>(a, L, st, sl, it, col0, rt, cs, acc); break;
            default: slice_bcq<4, NRT, NTILE, NMAT>(a, L, st, sl, it, col0, rt, cs, acc); break;
        }
    }
}

// ---------------------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------------------
template <int FMT, int NRT, int NTILE, int NMAT>
__global__ void __launch_bounds__(kVThreads, 1) vp_gemv_kernel(VpArgs a) {
    using Gm = Geo<NRT>;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t s_full[kMaxStages], s_empty[kMaxStages], s_slot_empty[2];
    __shared__ uint64_t s_red_full[NRT], s_red_free[NRT];
    __shared__ int s_abort;
    const VLayout L = vlayout<NRT, NTILE, NMAT>(a.K, a.G, FMT, a.B);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < L.nst; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], kCW);
        }
        for (int b = 0; b < 2; ++b) mbar_init(&s_slot_empty[b], kCW);
        for (int r = 0; r < NRT; ++r) {
            mbar_init(&s_red_full[r], Gm::CS - 1);
            mbar_init(&s_red_free[r], 1);
        }
        s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();   // work lists and activation digits come from the previous kernels
    volatile int* abort = &s_abort;
    const int K = a.K, ng = K / a.G;
    const int n_rb = a.R / Gm::RB;
    const int n_chunks = (K + Gm::CK - 1) / Gm::CK;
    const int n_items = static_cast<int>(__ldcg(&a.hdr->n_vgroups)) * n_rb;

    if (warp == kCW) {
        // ================================ producer ================================
        int q = 0;   // chunk counter over this CTA's items
        int issued_upto = 0;
        for (int n = 0, it = blockIdx.x; it < n_items && !*abort; ++n, it += gridDim.x) {
            const int slot = n & 1;
            unsigned char* sl = smem + L.nst * L.stage + slot * L.slot;
            if (n >= 2 && !vwait(&s_slot_empty[slot], ((n - 2) >> 1) & 1, abort, a.hdr, 0x301)) break;
            const int gi = it / n_rb, rb = it - gi * n_rb;
            const int4 grp = __ldcg(a.vgroups + gi);   // {e, kmax, ntiles, first tile}
            const int e = grp.x, kmax = grp.y, nt = grp.z;
            int4 tile = make_int4(0, 0, 0, 0);
            if (lane < nt) tile = __ldcg(a.vtiles + grp.w + lane);   // {k, pos0, n, 0}
            // token slots j = 4t + jj: digit row and output row of each
            const int tj = lane >> 2, jj = lane & 3;
            const int t_k = __shfl_sync(0xffffffffu, tile.x, tj & (NTILE - 1));
            const int t_pos0 = __shfl_sync(0xffffffffu, tile.y, tj & (NTILE - 1));
            const int t_n = __shfl_sync(0xffffffffu, tile.z, tj & (NTILE - 1));
            (void)t_k;
            int drow = -1, opos = -1;
            if (lane < 4 * NTILE && tj < nt && jj < t_n) {
                opos = t_pos0 + jj;
                drow = a.dig_by_token ? __ldcg(a.pos_tok + opos) : opos;
            }
            int* tab = reinterpret_cast<int*>(sl + L.sl_tab);
            if (lane == 0) {
                tab[0] = e;
                tab[1] = kmax;
                tab[2] = nt;
                tab[3] = rb;
            }
            if (lane < NTILE) {
                tab[4 + 4 * lane] = lane < nt ? tile.x : 0;
                tab[4 + 4 * lane + 1] = lane < nt ? tile.z : 0;
            }
            if (lane < 4 * NTILE) {
                tab[4 + 4 * NTILE + lane] = drow;
                tab[4 + 8 * NTILE + lane] = opos;
            }
            __syncwarp();
            const unsigned valid = __ballot_sync(0xffffffffu, drow >= 0);
            const uint8_t* pbase = a.planes + static_cast<uint64_t>(e) * a.planes_per_expert;
            const uint64_t plane_bytes = static_cast<uint64_t>(a.R) * K / 8;
            for (int c = 0; c < n_chunks; ++c, ++q) {
                const int s = q % L.nst;
                const int round = q / L.nst;
                if (round > 0 && !vwait(&s_empty[s], (round - 1) & 1, abort, a.hdr, 0x302)) goto producer_done;
                unsigned char* st = smem + s * L.stage;
                const int col0 = c * Gm::CK;
                const int cols = min(Gm::CK, K - col0);
                // bytes of this stage: planes, digits, and (first chunk) the slot's scales, exps, sums
                uint32_t bytes = static_cast<uint32_t>(NMAT * kmax * NRT) * (cols / 64) * 128u +
                                 static_cast<uint32_t>(__popc(valid)) * 2u * cols;
                const uint32_t mrow = FMT == DPA_FMT_UNIFORM ? static_cast<uint32_t>(Gm::RB * ng * 4)
                                                             : static_cast<uint32_t>(Gm::RB * ng * 2);
                const int n_meta = FMT == DPA_FMT_UNIFORM ? NMAT : NMAT * kmax;
                if (c == 0) bytes += n_meta * mrow + static_cast<uint32_t>(__popc(valid)) * 2u * L.ngp * 4u;
                if (lane == 0) {
                    fence_proxy_async();
                    mbar_arrive_expect_tx(&s_full[s], bytes);
                }
                __syncwarp();
                fence_proxy_async();
                // plane words: (m, p, rt) copies of cols/64 blocks
                const int n_pc = NMAT * kmax * NRT;
                for (int i = lane; i < n_pc; i += 32) {
                    const int rt = i % NRT, mp = i / NRT, p = mp % kmax, m = mp / kmax;
                    const uint8_t* src = pbase + a.planes_mat_off[a.mat0 + m] + p * plane_bytes +
                                         static_cast<uint64_t>(rb * NRT + rt) * (K / 64) * 128 +
                                         static_cast<uint64_t>(col0 / 64) * 128;
                    bulk_g2s(st + ((static_cast<size_t>(m * kMaxB + p) * NRT + rt) * (Gm::CK / 64)) * 128, src,
                             static_cast<uint32_t>(cols / 64) * 128u, &s_full[s]);
                }
                // digit rows of the tokens (two per token slot)
                if (lane < 4 * NTILE && drow >= 0) {
                    for (int d = 0; d < 2; ++d)
                        bulk_g2s(st + L.st_dig + static_cast<size_t>(lane * 2 + d) * L.dig_stride,
                                 a.dig + (static_cast<size_t>(drow) * 2 + d) * K + col0, static_cast<uint32_t>(cols),
                                 &s_full[s]);
                }
                if (c == 0) {
                    const uint8_t* mbase = a.meta + static_cast<uint64_t>(e) * a.meta_per_expert;
                    for (int i = lane; i < n_meta; i += 32) {
                        if (FMT == DPA_FMT_UNIFORM) {
                            bulk_g2s(sl + static_cast<size_t>(i) * mrow,
                                     mbase + a.meta_mat_off[a.mat0 + i] + static_cast<uint64_t>(rb) * mrow, mrow,
                                     &s_full[s]);
                        } else {
                            const int m = i / kmax, p = i % kmax;
                            bulk_g2s(sl + static_cast<size_t>(i) * mrow,
                                     mbase + a.meta_mat_off[a.mat0 + m] + static_cast<uint64_t>(p) * a.R * ng * 2 +
                                         static_cast<uint64_t>(rb) * mrow,
                                     mrow, &s_full[s]);
                        }
                    }
                    if (lane < 4 * NTILE && drow >= 0) {
                        bulk_g2s(sl + L.sl_exp + static_cast<size_t>(lane) * L.ngp * 4,
                                 a.dexp + static_cast<size_t>(drow) * L.ngp, static_cast<uint32_t>(L.ngp) * 4u,
                                 &s_full[s]);
                        bulk_g2s(sl + L.sl_sum + static_cast<size_t>(lane) * L.ngp * 4,
                                 a.dsum + static_cast<size_t>(drow) * L.ngp, static_cast<uint32_t>(L.ngp) * 4u,
                                 &s_full[s]);
                    }
                }
                issued_upto = q + 1;
            }
        }
    producer_done:
        // before the CTA exits every copy it issued must have landed: wait for the last stages
        for (int q2 = max(0, issued_upto - L.nst); q2 < issued_upto; ++q2) {
            const int s = q2 % L.nst;
            if (!mbar_try_wait(&s_full[s], (q2 / L.nst) & 1)) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait_suspend(&s_full[s], (q2 / L.nst) & 1, 10000u))
                    if (globaltimer() - t0 > kWaitNs) { set_error(a.hdr, DPA_ERR_DEVICE_TIMEOUT, 0x310); break; }
            }
        }
        return;
    }

    // ================================ consumers ================================
    const int rt = warp / Gm::CS, cs = warp % Gm::CS;
    int q = 0;
    for (int n = 0, it = blockIdx.x; it < n_items; ++n, it += gridDim.x) {
        const int slot = n & 1;
        const unsigned char* sl = smem + L.nst * L.stage + slot * L.slot;
        Item<NRT, NTILE, NMAT> item;
        float acc[NTILE][NMAT][2];
#pragma unroll
        for (int t = 0; t < NTILE; ++t)
#pragma unroll
            for (int m = 0; m < NMAT; ++m) acc[t][m][0] = acc[t][m][1] = 0.f;
        for (int c = 0; c < n_chunks; ++c, ++q) {
            const int s = q % L.nst;
            if (!vwait(&s_full[s], (q / L.nst) & 1, abort, a.hdr, 0x320)) return;
            if (c == 0) {
                const int* tab = reinterpret_cast<const int*>(sl + L.sl_tab);
                item.e = tab[0];
                item.kmax = tab[1];
                item.nt = tab[2];
                item.rb = tab[3];
#pragma unroll
                for (int t = 0; t < NTILE; ++t) {
                    item.tk[t] = tab[4 + 4 * t];
                    item.tn[t] = tab[4 + 4 * t + 1];
                }
            }
            slice_dispatch<FMT, NRT, NTILE, NMAT>(a, L, smem + s * L.stage, sl, item, c * Gm::CK, rt, cs, acc);
            __syncwarp();
            if (lane == 0) mbarrier_arrive(&s_empty[s]);
        }
        // ---- the column slices of this row tile meet (fixed order), then the epilogue ----
        // red_full completes once per item (the CS-1 slices arrive); red_free once per item (the
        // summing warp has read them), so a slice writes item n's partials after item n-1's read
        float* red = reinterpret_cast<float*>(smem + L.red);
        if (cs > 0) {
            if (n >= 1 && !vwait(&s_red_free[rt], (n - 1) & 1, abort, a.hdr, 0x330)) return;
            float* dst = red + (static_cast<size_t>(rt) * (Gm::CS - 1) + (cs - 1)) * (L.red_per / 4);
#pragma unroll
            for (int t = 0; t < NTILE; ++t)
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) dst[((t * NMAT + m) * 2 + rr) * 32 + lane] = acc[t][m][rr];
            __syncwarp();
            if (lane == 0) mbarrier_arrive(&s_red_full[rt]);
        } else {
            if (Gm::CS > 1 && !vwait(&s_red_full[rt], n & 1, abort, a.hdr, 0x331)) return;
            for (int c2 = 1; c2 < Gm::CS; ++c2) {
                const float* src = red + (static_cast<size_t>(rt) * (Gm::CS - 1) + (c2 - 1)) * (L.red_per / 4);
#pragma unroll
                for (int t = 0; t < NTILE; ++t)
#pragma unroll
                    for (int m = 0; m < NMAT; ++m)
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) acc[t][m][rr] += src[((t * NMAT + m) * 2 + rr) * 32 + lane];
            }
            __syncwarp();
            if (Gm::CS > 1 && lane == 0) mbarrier_arrive(&s_red_free[rt]);
            const int* tab = reinterpret_cast<const int*>(sl + L.sl_tab);
            const int gid = lane >> 2, tq = lane & 3;
#pragma unroll
            for (int t = 0; t < NTILE; ++t) {
                if (t < item.nt && tq < item.tn[t]) {
                    const int pos = tab[4 + 8 * NTILE + 4 * t + tq];
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int row = item.rb * Gm::RB + rt * 16 + gid + 8 * rr;
                        float v;
                        if constexpr (NMAT == 2) {
                            const float ag = acc[t][0][rr], au = acc[t][1][rr];
                            v = ag / (1.f + expf(-ag)) * au;
                        } else {
                            v = acc[t][0][rr];
                        }
                        a.out[static_cast<size_t>(pos) * a.R + row] = v;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbarrier_arrive(&s_slot_empty[slot]);
    }
}

// ---------------------------------------------------------------------------------------
// fixed-point digits of activation rows: bf16 tokens (x) or fp32 SwiGLU outputs (h)
// ---------------------------------------------------------------------------------------
// One warp per (row, group). Column c of a 64-column block is stored at byte
// 16*((c % 16) / 4) + 4*(c / 16) + c % 4 of the block, so that one 16-byte load gives a lane
// (tq = c % 16 / 4) its four B-operand words of the block.
__device__ __forceinline__ int perm64(int c) { return 16 * ((c & 15) >> 2) + 4 * (c >> 4) + (c & 3); }

template <bool BF16>
__global__ void __launch_bounds__(256) digits_kernel(DigitArgs d) {
    pdl_wait();
    const int K = d.K, G = d.G, ng = K / G, ngp = (ng + 3) & ~3;
    const int task = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (task >= d.rows * ng) return;
    const int r = task / ng, g = task - r * ng;
    float mx = 0.f;
    for (int j = lane; j < G; j += 32) {
        const float v = BF16 ? bf16_bits_to_float(d.x16[static_cast<size_t>(r) * K + g * G + j])
                             : d.x32[static_cast<size_t>(r) * K + g * G + j];
        mx = fmaxf(mx, fabsf(v));
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const int E = group_exponent(mx);
    int sum = 0;
    int8_t* d0row = d.dig + static_cast<size_t>(r) * 2 * K;
    int8_t* d1row = d0row + K;
    for (int j = lane; j < G; j += 32) {
        const int c = g * G + j;
        const float v = BF16 ? bf16_bits_to_float(d.x16[static_cast<size_t>(r) * K + c]) : d.x32[static_cast<size_t>(r) * K + c];
        const int X = __float2int_rn(ldexpf(v, 14 - E));
        sum += X;
        const int lo = ((X + 128) & 255) - 128;
        const int hi = (X - lo) >> 8;
        const int off = (c & ~63) + perm64(c & 63);
        d0row[off] = static_cast<int8_t>(lo);
        d1row[off] = static_cast<int8_t>(hi);
    }
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
        d.dexp[static_cast<size_t>(r) * ngp + g] = E;
        d.dsum[static_cast<size_t>(r) * ngp + g] = sum;
    }
}

template <int FMT, int NRT, int NTILE, int NMAT>
cudaError_t launch_variant(const VpArgs& a, cudaStream_t stream, int sms) {
    const VLayout L = vlayout<NRT, NTILE, NMAT>(a.K, a.G, FMT, a.B);
    const void* fn = reinterpret_cast<const void*>(vp_gemv_kernel<FMT, NRT, NTILE, NMAT>);
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
    if (err != cudaSuccess) return err;
    const int items = a.max_groups * (a.R / Geo<NRT>::RB);
    const int grid = items < sms ? (items > 0 ? items : 1) : sms;
    VpArgs copy = a;
    void* args[] = {&copy};
    return launch_pdl_raw(fn, dim3(grid), dim3(kVThreads), L.total, stream, args);
}

}  // namespace

size_t vp_smem_bytes(int K, int G, int fmt, int B, int nmat, bool multi) {
    if (nmat == 2)
        return multi ? vlayout<4, 2, 2>(K, G, fmt, B).total : vlayout<1, 1, 2>(K, G, fmt, B).total;
    return multi ? vlayout<4, 2, 1>(K, G, fmt, B).total : vlayout<4, 1, 1>(K, G, fmt, B).total;
}

cudaError_t launch_vp_gemv(const VpArgs& a, cudaStream_t stream, int sms) {
    if (a.nmat == 2) {
        if (a.fmt == DPA_FMT_UNIFORM)
            return a.multi ? launch_variant<DPA_FMT_UNIFORM, 4, 2, 2>(a, stream, sms)
                           : launch_variant<DPA_FMT_UNIFORM, 1, 1, 2>(a, stream, sms);
        return a.multi ? launch_variant<DPA_FMT_BCQ, 4, 2, 2>(a, stream, sms)
                       : launch_variant<DPA_FMT_BCQ, 1, 1, 2>(a, stream, sms);
    }
    if (a.fmt == DPA_FMT_UNIFORM)
        return a.multi ? launch_variant<DPA_FMT_UNIFORM, 4, 2, 1>(a, stream, sms)
                       : launch_variant<DPA_FMT_UNIFORM, 4, 1, 1>(a, stream, sms);
    return a.multi ? launch_variant<DPA_FMT_BCQ, 4, 2, 1>(a, stream, sms)
                   : launch_variant<DPA_FMT_BCQ, 4, 1, 1>(a, stream, sms);
}

cudaError_t launch_digits(const DigitArgs& d, cudaStream_t stream) {
    const int tasks = d.rows * (d.K / d.G);
    if (tasks <= 0) return cudaSuccess;
    DigitArgs copy = d;
    void* args[] = {&copy};
    const void* fn = d.x16 ? reinterpret_cast<const void*>(digits_kernel<true>)
                           : reinterpret_cast<const void*>(digits_kernel<false>);
    return launch_pdl_raw(fn, dim3((tasks + 7) / 8), dim3(256), 0, stream, args);
}

}  // namespace dpa
