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
// Work. A token group (written by the allocation as one record) is up to NTILE tiles of up to
// four pairs of one expert, each tile of one plane count k, tiles ascending in k. Items are
// (token group, block of RB = 16 NRT rows); every CTA (one per SM, persistent) takes a contiguous
// range of items, so consecutive items mostly share their group. Roles:
//   - warp CW (producer; CW = 12 consumer warps for uniform codes, 8 for binary-coded planes):
//     per group, bulk copies (no multicast) of the tokens' digit rows, group
//     exponents and sums into one of two group slots; per item and chunk of up to 2048 columns,
//     bulk copies of the chunk's plane words (one copy per matrix, plane p < kmax and row tile:
//     2 bytes per column) and, with the first chunk, the item's scale data into a ring stage;
//   - warps 0..CW-1 (consumers): row tile rt and column slice cs of every chunk (CW / NRT
//     slices per row tile); wait for the stage,
//     compute, release it; after the item's last chunk the slices of a row tile are summed in a
//     fixed order by one of them (rotating with the item) and the epilogue (SwiGLU for gate/up,
//     the per-pair output for down) is written.
// Every wait is bounded (globaltimer); on a timeout the kernel records DPA_ERR_DEVICE_TIMEOUT,
// sets a CTA-wide abort flag that ends every other wait, and the producer waits for the copies
// it issued before the CTA exits.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

// Consumer warps per CTA, by weight format. Uniform codes run 12: with the producer that is 13
// warps, so at most 4 share a scheduler and each thread keeps up to 128 registers, and the
// extra warps hide more of the decode's dependent latency (8 warps: 2 per scheduler). The
// binary-coded variants keep 8: their two-tile kernels need more than 128 registers.
#ifndef DPA_VP_CW_UNIFORM
#define DPA_VP_CW_UNIFORM 12
#endif
#ifndef DPA_VP_CW_BCQ
#define DPA_VP_CW_BCQ 8
#endif
__host__ __device__ constexpr int vp_cw(int fmt) { return fmt == DPA_FMT_UNIFORM ? DPA_VP_CW_UNIFORM : DPA_VP_CW_BCQ; }
constexpr int kMaxStages = 8;                 // ring depth: as many stages as shared memory holds
constexpr int kMaxB = 4;
#ifndef DPA_VP_CHUNK
#define DPA_VP_CHUNK 2048
#endif
constexpr int kMaxChunk = DPA_VP_CHUNK;       // columns per chunk
// Row tiles (16 rows each) per item: the larger where the ring and group slots fit in shared
// memory, else the smaller (wide matrices, whose scale data and digit rows take more room).
#ifndef DPA_VP_GU_NRT_UNIFORM
#define DPA_VP_GU_NRT_UNIFORM 4
#endif
#ifndef DPA_VP_GU_NRT_BCQ
#define DPA_VP_GU_NRT_BCQ 2
#endif
#ifndef DPA_VP_DN_NRT
#define DPA_VP_DN_NRT 4
#endif
// gate/up: 64 rows (uniform codes, 3 column slices of the 12 consumer warps) or 32 rows
// (binary-coded planes, 4 slices of 8), else 16 rows
constexpr int kGuNRTUniform = DPA_VP_GU_NRT_UNIFORM, kGuNRTBcq = DPA_VP_GU_NRT_BCQ, kGuNRTSmall = 1;
constexpr int kDnNRT = DPA_VP_DN_NRT, kDnNRTSmall = 2;   // down: 64 (32) rows, 2 (4) column slices
constexpr int kDigPad = 64;                   // bytes of padding per staged digit row (banks)

template <int CW, int NRT>
struct Geo {
    static_assert(CW % NRT == 0, "the consumer warps split into row tiles x column slices");
    static constexpr int CS = CW / NRT;       // column slices per chunk
    static constexpr int RB = 16 * NRT;       // rows per item
};

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~static_cast<size_t>(15); }
__host__ __device__ inline size_t al128(size_t v) { return (v + 127) & ~static_cast<size_t>(127); }

struct VLayout {                              // byte offsets in dynamic shared memory (< 227 KB)
    uint32_t CK;                              // columns per chunk
    uint32_t stage, st_meta;                  // per stage: planes at 0, then the item's scale data
    uint32_t slot, sl_exp, sl_sum, sl_rec;    // per group slot: digits at 0, scales, scaled sums, record
    uint32_t dig_stride;                      // bytes per staged digit row (K + pad)
    uint32_t slots, red, red_per;             // group slots' offset; reduction buffer
    uint32_t total;
    int nst;                                  // stages in the ring
    int ngp;                                  // exps/sums row stride (ints)
};

template <int NRT, int NTILE, int NMAT>
__host__ __device__ inline VLayout vlayout(int K, int G, int fmt, int B) {
    constexpr int RB = 16 * NRT;
    const int CS = vp_cw(fmt) / NRT;
    VLayout L;
    const size_t ng = K / G;
    L.ngp = static_cast<int>((ng + 3) & ~static_cast<size_t>(3));
    const size_t meta = fmt == DPA_FMT_UNIFORM ? static_cast<size_t>(NMAT) * RB * ng * 4
                                               : static_cast<size_t>(NMAT) * B * RB * ng * 2;
    const size_t dig_stride = static_cast<size_t>(K) + kDigPad;
    const size_t digs = static_cast<size_t>(4 * NTILE) * 2 * dig_stride;
    const size_t sl_exp = al16(digs);
    const size_t sl_sum = sl_exp + static_cast<size_t>(4 * NTILE) * L.ngp * 4;
    const size_t sl_rec = sl_sum + static_cast<size_t>(4 * NTILE) * L.ngp * 4;
    const size_t slot = al128(sl_rec + kVRecInts * 4);
    const size_t red_per = static_cast<size_t>(32) * NTILE * NMAT * 2 * 4;
    const size_t red = static_cast<size_t>(NRT) * CS * red_per;   // one partial per warp
    const size_t fixed = 2 * slot + red;
    // columns per chunk: every column (one copy per matrix and plane takes all the item's row
    // tiles) where two stages fit beside the fixed parts, else halved down to 512
    size_t CK = K < kMaxChunk ? K : kMaxChunk, planes = 0, stage = 0;
    for (;;) {
        planes = static_cast<size_t>(NMAT) * kMaxB * NRT * (CK / 64) * 128;
        stage = al128(planes + al16(meta));
        if (fixed + 2 * stage <= kVpMaxSmem || CK <= 512 || (CK / 2) % 64 != 0) break;
        CK /= 2;
    }
    int nst = 2;   // at least double buffering; more while the ring fits beside the fixed parts
    while (nst < kMaxStages && fixed + (nst + 1) * stage <= kVpMaxSmem) ++nst;
    size_t total = nst * stage + fixed;
    if (total > 0xFFFFFFFFull) total = 0xFFFFFFFFull;   // rejected by the caller (too large)
    L.CK = static_cast<uint32_t>(CK);
    L.stage = static_cast<uint32_t>(stage);
    L.st_meta = static_cast<uint32_t>(planes);
    L.slot = static_cast<uint32_t>(slot);
    L.sl_exp = static_cast<uint32_t>(sl_exp);
    L.sl_sum = static_cast<uint32_t>(sl_sum);
    L.sl_rec = static_cast<uint32_t>(sl_rec);
    L.dig_stride = static_cast<uint32_t>(dig_stride);
    L.slots = static_cast<uint32_t>(nst * stage);
    L.red = static_cast<uint32_t>(nst * stage + 2 * slot);
    L.red_per = static_cast<uint32_t>(red_per);
    L.total = static_cast<uint32_t>(total);
    L.nst = nst;
    return L;
}

// waits that end on a bounded time or on the CTA's abort flag
__device__ __forceinline__ bool vwait(uint64_t* bar, uint32_t parity, volatile int* abort, WsHeader* hdr,
                                      uint32_t where) {
    return mbar_wait_abortable(bar, parity, abort, hdr, where);
}

// ---- uniform codes: plane merge (the plane layout of layout.h: in plane p, position rho of
// nibble m sits at bit 4m + (B-1-p) - rho, mod 32) ----
// The words of planes [0, KM) merged with fixed masks: bit (4m + T - RHO) mod 32 comes from the
// plane whose code bit is T. Rotating the result left by RHO gives the register of 8 codes of
// position RHO (nibble m = code m); positions of planes >= KM hold plane 0's bits, which the
// level mask of a k <= KM read removes.
template <int B, int KM, int RHO>
__device__ __forceinline__ uint32_t merge_planes(const uint32_t (&w)[kMaxB]) {
    uint32_t x = w[0];
#pragma unroll
    for (int p = 1; p < KM; ++p) {
        const uint32_t M = 0x11111111u << ((B - 1 - p - RHO) & 3);
        x = (x & ~M) | (w[p] & M);
    }
    return x;
}
__device__ __forceinline__ uint32_t rotl(uint32_t x, int s) { return __funnelshift_l(x, x, s); }
__device__ __forceinline__ uint32_t rotr(uint32_t x, int s) { return __funnelshift_r(x, x, s); }
// Codes of position rho, unmasked: lo[rho] holds nibble 2b in the low half of byte b, hi[rho]
// nibble 2b+1 (the A bytes of the block's first and second 32-column MMA).
template <int B, int KM>
__device__ __forceinline__ void decode_uniform(uint32_t (&lo)[4], uint32_t (&hi)[4], const uint32_t (&w)[kMaxB]) {
    const uint32_t x0 = merge_planes<B, KM, 0>(w), x1 = merge_planes<B, KM, 1>(w);
    const uint32_t x2 = merge_planes<B, KM, 2>(w), x3 = merge_planes<B, KM, 3>(w);
    lo[0] = x0;
    hi[0] = rotr(x0, 4);
    lo[1] = rotl(x1, 1);
    hi[1] = rotr(x1, 3);
    lo[2] = rotl(x2, 2);
    hi[2] = rotr(x2, 2);
    lo[3] = rotl(x3, 3);
    hi[3] = rotr(x3, 1);
}
// the codes of a k-plane read: the top k of B bits of every nibble, in the low nibble of a byte
__host__ __device__ inline uint32_t level_mask(int B, int k) {
    const uint32_t nib = ((1u << k) - 1u) << (B - k);
    return 0x0F0F0F0Fu & (nib * 0x01010101u);
}

// ---- B operand: the lane's 16 digit bytes of one 64-column block (one 16-byte load) ----
__device__ __forceinline__ uint4 lds128(const unsigned char* p) { return *reinterpret_cast<const uint4*>(p); }

// the group of the current item, as the consumers read it from the group slot's record
template <int NTILE>
struct Group {
    int kmax, nt;
    int tk[NTILE], tn[NTILE];
    uint32_t mk[NTILE];   // uniform codes: level mask of the tile's plane count
    float ck[NTILE];      // uniform codes: compensation constant c_k = (2^(B-k) - 1) / 2
};

// Where a slice's blocks fall in the scale groups: the first block's group and its index in
// the group (one division per slice; the block loop only counts).
struct SlicePos {
    int g, j;
};
__device__ __forceinline__ SlicePos slice_pos(int col0, int b0, int bpg) {
    const int blk = col0 / 64 + b0;
    SlicePos sp;
    sp.g = blk / bpg;
    sp.j = blk - sp.g * bpg;
    return sp;
}

// ---------------------------------------------------------------------------------------
// consumer: one column slice of one chunk, uniform codes, KM = the group's kmax planes and NT
// token tiles (both compile-time here). Blocks [b0, b1) of the chunk; the group slot holds the
// tokens' digits for every column (col0 = the chunk's first column). Per scale-group portion:
// int32 MMA accumulation, then one fp32 epilogue
//   acc += s * (f v + (c_k - z) f SX)   [the SX term once per group: in its first block's slice]
// with f = 2^(E-14) and f SX read from the slot.
// ---------------------------------------------------------------------------------------
template <int B, int KM, int NT, int NRT, int NTILE, int NMAT>
__device__ __forceinline__ void slice_uniform(const VpArgs& a, const VLayout& L, const unsigned char* st,
                                              const unsigned char* gs, const Group<NTILE>& gr, int col0, int b0,
                                              int b1, int rt, float (&acc)[NTILE][NMAT][2]) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tq = lane & 3;
    const int ng = a.K / a.G, bpg = a.G / 64, nbc = L.CK / 64;
    const int pstride = NRT * nbc * 32;                                   // words per (matrix, plane) slab
    const uint32_t* pw = reinterpret_cast<const uint32_t*>(st) + rt * nbc * 32 + lane;
    const uint32_t* mrow = reinterpret_cast<const uint32_t*>(st + L.st_meta) + (rt * 16 + gid) * ng;
    const float* fscl = reinterpret_cast<const float*>(gs + L.sl_exp) + tq * L.ngp;
    const float* ffsx = reinterpret_cast<const float*>(gs + L.sl_sum) + tq * L.ngp;
    const unsigned char* bsrc = gs + static_cast<size_t>((gid >> 1) * 2 + (gid & 1)) * L.dig_stride + 16 * tq + col0;
    SlicePos sp = slice_pos(col0, b0, bpg);
    int cb = b0;
#pragma unroll 1
    while (cb < b1) {
        const int n = min(bpg - sp.j, b1 - cb);   // blocks of this group portion
        const bool has_start = sp.j == 0;
        int C[NT][NMAT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int m = 0; m < NMAT; ++m) C[t][m][0] = C[t][m][1] = C[t][m][2] = C[t][m][3] = 0;
#pragma unroll 1
        for (int i = 0; i < n; ++i, ++cb) {
            uint4 bt[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) bt[t] = lds128(bsrc + static_cast<size_t>(8 * t) * L.dig_stride + cb * 64);
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                uint32_t w[kMaxB];
#pragma unroll
                for (int p = 0; p < kMaxB; ++p) w[p] = p < KM ? pw[(m * kMaxB + p) * pstride + cb * 32] : 0u;
                uint32_t R[4], Rh[4];
                decode_uniform<B, KM>(R, Rh, w);
                uint32_t Alo[4], Ahi[4];
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (t == 0 || gr.mk[t] != gr.mk[t - 1]) {
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            Alo[r] = R[r] & gr.mk[t];
                            Ahi[r] = Rh[r] & gr.mk[t];
                        }
                    }
                    mma_u8s8(C[t][m], Alo[0], Alo[1], Alo[2], Alo[3], bt[t].x, bt[t].y);
                    mma_u8s8(C[t][m], Ahi[0], Ahi[1], Ahi[2], Ahi[3], bt[t].z, bt[t].w);
                }
            }
        }
        // ---- epilogue of the portion of group g ----
        const int g = sp.g;
        float s[NMAT][2], z[NMAT][2];
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const uint32_t sz = mrow[(m * 16 * NRT + 8 * rr) * ng + g];
                s[m][rr] = __half2float(__ushort_as_half(static_cast<unsigned short>(sz & 0xFFFFu)));
                z[m][rr] = __half2float(__ushort_as_half(static_cast<unsigned short>(sz >> 16)));
            }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float f = fscl[4 * t * L.ngp + g];
            const float fsx = has_start ? ffsx[4 * t * L.ngp + g] : 0.f;
            const float a0 = gr.ck[t] * fsx;
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const float v = static_cast<float>(C[t][m][2 * rr] + 256 * C[t][m][2 * rr + 1]);
                    const float u = fmaf(-z[m][rr], fsx, fmaf(f, v, a0));
                    acc[t][m][rr] = fmaf(s[m][rr], u, acc[t][m][rr]);
                }
        }
        sp.j = 0;
        ++sp.g;
    }
}

// ---------------------------------------------------------------------------------------
// consumer: one column slice of one chunk, binary-coded planes (KM planes, NT tiles):
//   acc += alpha_p (2 f S_p - f SX)   per plane p < k of the tile and group portion
// ---------------------------------------------------------------------------------------
template <int B, int KM, int NT, int NRT, int NTILE, int NMAT>
__device__ __forceinline__ void slice_bcq(const VpArgs& a, const VLayout& L, const unsigned char* st,
                                          const unsigned char* gs, const Group<NTILE>& gr, int col0, int b0, int b1,
                                          int rt, float (&acc)[NTILE][NMAT][2]) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tq = lane & 3;
    const int ng = a.K / a.G, bpg = a.G / 64, nbc = L.CK / 64;
    const int pstride = NRT * nbc * 32;
    const uint32_t* pw = reinterpret_cast<const uint32_t*>(st) + rt * nbc * 32 + lane;
    const __half* meta = reinterpret_cast<const __half*>(st + L.st_meta);
    const float* fscl = reinterpret_cast<const float*>(gs + L.sl_exp) + tq * L.ngp;
    const float* ffsx = reinterpret_cast<const float*>(gs + L.sl_sum) + tq * L.ngp;
    const unsigned char* bsrc = gs + static_cast<size_t>((gid >> 1) * 2 + (gid & 1)) * L.dig_stride + 16 * tq + col0;
    SlicePos sp = slice_pos(col0, b0, bpg);
    int cb0 = b0;
#pragma unroll 1
    while (cb0 < b1) {
        const int n = min(bpg - sp.j, b1 - cb0);
        const bool has_start = sp.j == 0;
        const int g = sp.g;
#pragma unroll 1
        for (int p = 0; p < KM; ++p) {
            int C[NT][NMAT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int m = 0; m < NMAT; ++m) C[t][m][0] = C[t][m][1] = C[t][m][2] = C[t][m][3] = 0;
#pragma unroll 1
            for (int i = 0; i < n; ++i) {
                const int cb = cb0 + i;
                uint4 bt[NT];
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    if (gr.tk[t] > p) bt[t] = lds128(bsrc + static_cast<size_t>(8 * t) * L.dig_stride + cb * 64);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const uint32_t w = pw[(m * kMaxB + p) * pstride + cb * 32];
                    uint32_t lo[4], hi[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        lo[r] = (w >> r) & 0x01010101u;
                        hi[r] = (w >> (r + 4)) & 0x01010101u;
                    }
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        if (gr.tk[t] > p) {
                            mma_u8s8(C[t][m], lo[0], lo[1], lo[2], lo[3], bt[t].x, bt[t].y);
                            mma_u8s8(C[t][m], hi[0], hi[1], hi[2], hi[3], bt[t].z, bt[t].w);
                        }
                    }
                }
            }
            float al[NMAT][2];
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int rr = 0; rr < 2; ++rr)
                    al[m][rr] = __half2float(meta[((m * KM + p) * 16 * NRT + rt * 16 + gid + 8 * rr) * ng + g]);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (gr.tk[t] > p) {
                    const float f2 = 2.f * fscl[4 * t * L.ngp + g];
                    const float fsx = has_start ? ffsx[4 * t * L.ngp + g] : 0.f;
#pragma unroll
                    for (int m = 0; m < NMAT; ++m)
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            const float v = static_cast<float>(C[t][m][2 * rr] + 256 * C[t][m][2 * rr + 1]);
                            acc[t][m][rr] = fmaf(al[m][rr], fmaf(f2, v, -fsx), acc[t][m][rr]);
                        }
                }
            }
        }
        cb0 += n;
        sp.j = 0;
        ++sp.g;
    }
}

// one slice with the group's plane count and tile count as compile-time constants
template <int FMT, int B, int NRT, int NTILE, int NMAT>
__device__ __forceinline__ void slice_b(const VpArgs& a, const VLayout& L, const unsigned char* st,
                                        const unsigned char* gs, const Group<NTILE>& gr, int col0, int b0, int b1,
                                        int rt, float (&acc)[NTILE][NMAT][2]) {
#define DPA_SLICE(KM, NT)                                                                                 \
    do {                                                                                                  \
        if constexpr (FMT == DPA_FMT_UNIFORM)                                                             \
            slice_uniform<B, KM, NT, NRT, NTILE, NMAT>(a, L, st, gs, gr, col0, b0, b1, rt, acc);           \
        else                                                                                              \
            slice_bcq<B, KM, NT, NRT, NTILE, NMAT>(a, L, st, gs, gr, col0, b0, b1, rt, acc);               \
    } while (0)
    const int km = gr.kmax;
    if (NTILE == 1 || gr.nt == 1) {
        if (km == 1) DPA_SLICE(1, 1);
        else if (km == 2 && B >= 2) DPA_SLICE(2 <= B ? 2 : B, 1);
        else if (km == 3 && B >= 3) DPA_SLICE(3 <= B ? 3 : B, 1);
        else DPA_SLICE(B, 1);
    } else {
        constexpr int NT2 = NTILE >= 2 ? 2 : 1;
        if (km == 1) DPA_SLICE(1, NT2);
        else if (km == 2 && B >= 2) DPA_SLICE(2 <= B ? 2 : B, NT2);
        else if (km == 3 && B >= 3) DPA_SLICE(3 <= B ? 3 : B, NT2);
        else DPA_SLICE(B, NT2);
    }
#undef DPA_SLICE
}

template <int FMT, int NRT, int NTILE, int NMAT>
__device__ __forceinline__ void slice_dispatch(const VpArgs& a, const VLayout& L, const unsigned char* st,
                                               const unsigned char* gs, const Group<NTILE>& gr, int col0, int b0,
                                               int b1, int rt, float (&acc)[NTILE][NMAT][2]) {
    switch (a.B) {
        case 1: slice_b<FMT, 1, NRT, NTILE, NMAT>(a, L, st, gs, gr, col0, b0, b1, rt, acc); break;
        case 2: slice_b<FMT, 2, NRT, NTILE, NMAT>(a, L, st, gs, gr, col0, b0, b1, rt, acc); break;
        case 3: slice_b<FMT, 3, NRT, NTILE, NMAT>(a, L, st, gs, gr, col0, b0, b1, rt, acc); break;
        default: slice_b<FMT, 4, NRT, NTILE, NMAT>(a, L, st, gs, gr, col0, b0, b1, rt, acc); break;
    }
}

// ---------------------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------------------
template <int FMT, int NRT, int NTILE, int NMAT>
__global__ void __launch_bounds__((vp_cw(FMT) + 1) * 32, 1) vp_gemv_kernel(VpArgs a) {
    constexpr int kCW = vp_cw(FMT);   // consumer warps; warp kCW is the producer
    using Gm = Geo<kCW, NRT>;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t s_full[kMaxStages], s_empty[kMaxStages], s_gfull[2], s_gempty[2];
    // the reduction's "partials written" barrier alternates with the item's parity: warps run up
    // to a ring's depth apart, so when an item's reducer arrives one shared barrier could be in
    // the previous item's phase, this one's, or the next one's, which a parity wait cannot tell
    // apart; with two, each is at most one phase from the one awaited
    __shared__ uint64_t s_red_full[NRT][2], s_red_free[NRT];
    __shared__ int s_abort;
    const VLayout L = vlayout<NRT, NTILE, NMAT>(a.K, a.G, FMT, a.B);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < L.nst; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], kCW);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_gfull[b], 1);
            mbar_init(&s_gempty[b], kCW);
        }
        for (int r = 0; r < NRT; ++r) {
            mbar_init(&s_red_full[r][0], Gm::CS - 1);
            mbar_init(&s_red_full[r][1], Gm::CS - 1);
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
    const int n_chunks = (K + static_cast<int>(L.CK) - 1) / static_cast<int>(L.CK);
    const int n_items = static_cast<int>(__ldcg(&a.hdr->n_vgroups)) * n_rb;
    // this CTA's contiguous range of items
    int it0 = static_cast<int>((static_cast<long long>(n_items) * blockIdx.x) / gridDim.x);
    int it1 = static_cast<int>((static_cast<long long>(n_items) * (blockIdx.x + 1)) / gridDim.x);
    if (a.vstart && a.vgrid == static_cast<int>(gridDim.x) && n_items > 2 * static_cast<int>(gridDim.x)) {
        // ranges balanced by the groups' estimated work (written for batches with more than two
        // items per CTA)
        it0 = min(__ldcg(a.vstart + blockIdx.x), n_items);
        it1 = min(__ldcg(a.vstart + blockIdx.x + 1), n_items);
    }

    if (warp == kCW) {
        // ================================ producer ================================
        int q = 0, gcount = 0, cur_g = -1, kmax = 0, e = 0;
        int issued_upto = 0, groups_issued = 0;
        const uint32_t mrow = FMT == DPA_FMT_UNIFORM ? static_cast<uint32_t>(Gm::RB * ng * 4)
                                                     : static_cast<uint32_t>(Gm::RB * ng * 2);
        const uint64_t plane_bytes = static_cast<uint64_t>(a.R) * K / 8;
        for (int it = it0; it < it1 && !*abort; ++it) {
            const int gi = it / n_rb, rb = it - gi * n_rb;
            if (gi != cur_g) {
                // ---- a new token group: its record, digit rows, exponents and sums -> group slot
                const int slot = gcount & 1;
                if (gcount >= 2 && !vwait(&s_gempty[slot], ((gcount - 2) >> 1) & 1, abort, a.hdr, 0x301)) break;
                const int rv = __ldcg(a.vrec + static_cast<size_t>(gi) * kVRecInts + lane);
                e = __shfl_sync(0xffffffffu, rv, 0);
                kmax = __shfl_sync(0xffffffffu, rv, 1);
                const int drow = __shfl_sync(0xffffffffu, rv, (a.dig_by_token ? 16 : 8) + (lane & 7));
                const bool valid = lane < 4 * NTILE && drow >= 0;
                unsigned char* gs = smem + L.slots + slot * L.slot;
                reinterpret_cast<int*>(gs + L.sl_rec)[lane] = rv;
                __syncwarp();
                const uint32_t nvalid = static_cast<uint32_t>(__popc(__ballot_sync(0xffffffffu, valid)));
                if (lane == 0) {
                    fence_proxy_async();
                    mbar_arrive_expect_tx(&s_gfull[slot], nvalid * (2u * K + 2u * L.ngp * 4u));
                }
                __syncwarp();
                fence_proxy_async();
                if (valid) {
                    for (int d = 0; d < 2; ++d)
                        bulk_g2s(gs + static_cast<size_t>(lane * 2 + d) * L.dig_stride,
                                 a.dig + (static_cast<size_t>(drow) * 2 + d) * K, static_cast<uint32_t>(K), &s_gfull[slot]);
                    bulk_g2s(gs + L.sl_exp + static_cast<size_t>(lane) * L.ngp * 4,
                             a.dscl + static_cast<size_t>(drow) * L.ngp, static_cast<uint32_t>(L.ngp) * 4u, &s_gfull[slot]);
                    bulk_g2s(gs + L.sl_sum + static_cast<size_t>(lane) * L.ngp * 4,
                             a.dfsx + static_cast<size_t>(drow) * L.ngp, static_cast<uint32_t>(L.ngp) * 4u, &s_gfull[slot]);
                }
                cur_g = gi;
                ++gcount;
                groups_issued = gcount;
            }
            // the expert's planes and scale data: the full layout, or the compact layer of
            // per-expert stored widths (expert e holds w_e planes per matrix at its own offsets)
            const uint8_t* pbase;
            const uint8_t* mbase;
            uint64_t pmat[NMAT], mplane = static_cast<uint64_t>(a.R) * ng * 2;   // BCQ alphas per plane
            uint64_t mmat[NMAT];
            if (a.expert_off) {
                const uint64_t w = __ldg(a.expert_width + e);
                pbase = a.planes + __ldg(a.expert_off + 2 * e);
                mbase = a.meta + __ldg(a.expert_off + 2 * e + 1);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    pmat[m] = (a.mat0 + m) * w * plane_bytes;
                    mmat[m] = FMT == DPA_FMT_UNIFORM ? a.meta_mat_off[a.mat0 + m] : (a.mat0 + m) * w * mplane;
                }
            } else {
                pbase = a.planes + static_cast<uint64_t>(e) * a.planes_per_expert;
                mbase = a.meta + static_cast<uint64_t>(e) * a.meta_per_expert;
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    pmat[m] = a.planes_mat_off[a.mat0 + m];
                    mmat[m] = a.meta_mat_off[a.mat0 + m];
                }
            }
            const int n_meta = FMT == DPA_FMT_UNIFORM ? NMAT : NMAT * kmax;
            for (int c = 0; c < n_chunks; ++c, ++q) {
                const int s = q % L.nst;
                const int round = q / L.nst;
                if (round > 0 && !vwait(&s_empty[s], (round - 1) & 1, abort, a.hdr, 0x302)) goto producer_done;
                unsigned char* st = smem + s * L.stage;
                const int col0 = c * static_cast<int>(L.CK);
                const int cols = min(static_cast<int>(L.CK), K - col0);
                const int n_pc = NMAT * kmax * NRT;
                const uint32_t bytes = static_cast<uint32_t>(n_pc) * (cols / 64) * 128u + n_meta * mrow;
                if (lane == 0) {
                    fence_proxy_async();
                    mbar_arrive_expect_tx(&s_full[s], bytes);
                }
                __syncwarp();
                fence_proxy_async();
                // plane words: (m, p, rt) copies of the chunk's columns (2 bytes per column); a chunk
                // of every column takes the item's NRT consecutive row tiles in one copy per (m, p)
                if (static_cast<int>(L.CK) == K) {
                    for (int i = lane; i < NMAT * kmax; i += 32) {
                        const int p = i % kmax, m = i / kmax;
                        const uint8_t* src = pbase + pmat[m] + p * plane_bytes +
                                             static_cast<uint64_t>(rb * NRT) * (K / 64) * 128;
                        bulk_g2s(st + (static_cast<size_t>(m * kMaxB + p) * NRT * (K / 64)) * 128, src,
                                 static_cast<uint32_t>(NRT * (K / 64)) * 128u, &s_full[s]);
                    }
                } else
                for (int i = lane; i < n_pc; i += 32) {
                    const int rt = i % NRT, mp = i / NRT, p = mp % kmax, m = mp / kmax;
                    const uint8_t* src = pbase + pmat[m] + p * plane_bytes +
                                         static_cast<uint64_t>(rb * NRT + rt) * (K / 64) * 128 +
                                         static_cast<uint64_t>(col0 / 64) * 128;
                    bulk_g2s(st + ((static_cast<size_t>(m * kMaxB + p) * NRT + rt) * (L.CK / 64)) * 128, src,
                             static_cast<uint32_t>(cols / 64) * 128u, &s_full[s]);
                }
                // the item's scale data (every stage carries it, for the chunks that follow)
                for (int i = lane; i < n_meta; i += 32) {
                    const uint8_t* src;
                    if (FMT == DPA_FMT_UNIFORM) {
                        src = mbase + mmat[i] + static_cast<uint64_t>(rb) * mrow;
                    } else {
                        const int m = i / kmax, p = i % kmax;
                        src = mbase + mmat[m] + static_cast<uint64_t>(p) * mplane +
                              static_cast<uint64_t>(rb) * mrow;
                    }
                    bulk_g2s(st + L.st_meta + static_cast<size_t>(i) * mrow, src, mrow, &s_full[s]);
                }
                issued_upto = q + 1;
            }
        }
    producer_done:
        // before the CTA exits every copy it issued must have landed: the last stages and groups
        for (int q2 = max(0, issued_upto - L.nst); q2 < issued_upto; ++q2) {
            const int s = q2 % L.nst;
            if (!mbar_try_wait(&s_full[s], (q2 / L.nst) & 1)) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait_suspend(&s_full[s], (q2 / L.nst) & 1, 10000u))
                    if (globaltimer() - t0 > kWaitNs) { set_error(a.hdr, DPA_ERR_DEVICE_TIMEOUT, 0x310); break; }
            }
        }
        for (int g2 = max(0, groups_issued - 2); g2 < groups_issued; ++g2) {
            const int slot = g2 & 1;
            if (!mbar_try_wait(&s_gfull[slot], (g2 >> 1) & 1)) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait_suspend(&s_gfull[slot], (g2 >> 1) & 1, 10000u))
                    if (globaltimer() - t0 > kWaitNs) { set_error(a.hdr, DPA_ERR_DEVICE_TIMEOUT, 0x311); break; }
            }
        }
        return;
    }

    // ================================ consumers ================================
    const int rt = warp / Gm::CS, cs = warp % Gm::CS;
    const int gid = lane >> 2, tq = lane & 3;
    float* red = reinterpret_cast<float*>(smem + L.red);
    int q = 0, gcount = 0, cur_g = -1, ni = 0;
    const unsigned char* gs = nullptr;
    Group<NTILE> gr;
    for (int it = it0; it < it1; ++it, ++ni) {
        const int gi = it / n_rb, rb = it - gi * n_rb;
        if (gi != cur_g) {
            if (cur_g >= 0) {   // the previous group's slot is no longer read
                __syncwarp();
                if (lane == 0) mbarrier_arrive(&s_gempty[(gcount - 1) & 1]);
            }
            const int slot = gcount & 1;
            if (!vwait(&s_gfull[slot], (gcount >> 1) & 1, abort, a.hdr, 0x321)) return;
            gs = smem + L.slots + slot * L.slot;
            const int* rec = reinterpret_cast<const int*>(gs + L.sl_rec);
            gr.kmax = rec[1];
            gr.nt = rec[2];
#pragma unroll
            for (int t = 0; t < NTILE; ++t) {
                gr.tk[t] = rec[4 + t];
                gr.tn[t] = rec[6 + t];
                const int k = gr.tk[t] > 0 ? gr.tk[t] : 1;
                gr.mk[t] = level_mask(a.B, k);
                gr.ck[t] = 0.5f * static_cast<float>((1 << (a.B - k)) - 1);
            }
            cur_g = gi;
            ++gcount;
        }
        float acc[NTILE][NMAT][2];
#pragma unroll
        for (int t = 0; t < NTILE; ++t)
#pragma unroll
            for (int m = 0; m < NMAT; ++m) acc[t][m][0] = acc[t][m][1] = 0.f;
        for (int c = 0; c < n_chunks; ++c, ++q) {
            const int s = q % L.nst;
            if (!vwait(&s_full[s], (q / L.nst) & 1, abort, a.hdr, 0x320)) return;
            const int col0 = c * static_cast<int>(L.CK);
            const int nbc = min(static_cast<int>(L.CK), K - col0) / 64;
            const int b0 = (cs * nbc) / Gm::CS, b1 = ((cs + 1) * nbc) / Gm::CS;
            slice_dispatch<FMT, NRT, NTILE, NMAT>(a, L, smem + s * L.stage, gs, gr, col0, b0, b1, rt, acc);
            __syncwarp();
            if (lane == 0) mbarrier_arrive(&s_empty[s]);
        }
        // ---- the column slices of this row tile meet: one of them (rotating with the item)
        // sums the partials in slice order and writes the epilogue ----
        const int reducer = ni % Gm::CS;
        float* part = red + static_cast<size_t>(rt * Gm::CS) * (L.red_per / 4);
        if (cs != reducer) {
            // the previous item's reducer must have read its partials before they are rewritten
            if (ni >= 1 && !vwait(&s_red_free[rt], (ni - 1) & 1, abort, a.hdr, 0x330)) return;
            float* dst = part + static_cast<size_t>(cs) * (L.red_per / 4);
#pragma unroll
            for (int t = 0; t < NTILE; ++t)
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) dst[((t * NMAT + m) * 2 + rr) * 32 + lane] = acc[t][m][rr];
            __syncwarp();
            if (lane == 0) mbarrier_arrive(&s_red_full[rt][ni & 1]);
        } else {
            if (Gm::CS > 1 && !vwait(&s_red_full[rt][ni & 1], (ni >> 1) & 1, abort, a.hdr, 0x331)) return;
            float sum[NTILE][NMAT][2];
#pragma unroll
            for (int t = 0; t < NTILE; ++t)
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) sum[t][m][rr] = 0.f;
            for (int c2 = 0; c2 < Gm::CS; ++c2) {   // fixed order: slice 0, 1, ...
                const float* src = part + static_cast<size_t>(c2) * (L.red_per / 4);
#pragma unroll
                for (int t = 0; t < NTILE; ++t)
#pragma unroll
                    for (int m = 0; m < NMAT; ++m)
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr)
                            sum[t][m][rr] += c2 == cs ? acc[t][m][rr] : src[((t * NMAT + m) * 2 + rr) * 32 + lane];
            }
            __syncwarp();
            if (Gm::CS > 1 && lane == 0) mbarrier_arrive(&s_red_free[rt]);
            const int* rec = reinterpret_cast<const int*>(gs + L.sl_rec);
#pragma unroll
            for (int t = 0; t < NTILE; ++t) {
                if (t < gr.nt && tq < gr.tn[t]) {
                    const int pos = rec[8 + 4 * t + tq];
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int row = rb * Gm::RB + rt * 16 + gid + 8 * rr;
                        float v;
                        if constexpr (NMAT == 2) {
                            const float ag = sum[t][0][rr], au = sum[t][1][rr];
                            v = ag / (1.f + expf(-ag)) * au;
                        } else {
                            v = sum[t][0][rr];
                        }
                        a.out[static_cast<size_t>(pos) * a.R + row] = v;
                    }
                }
            }
        }
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
    if (lane == 0) {   // |sum| <= G 2^14 <= 2^23: the scaled sum is exact in fp32
        const float scl = ldexpf(1.f, E - 14);
        d.dscl[static_cast<size_t>(r) * ngp + g] = scl;
        d.dfsx[static_cast<size_t>(r) * ngp + g] = scl * static_cast<float>(sum);
    }
}

template <int FMT, int NRT, int NTILE, int NMAT>
cudaError_t launch_variant(const VpArgs& a, cudaStream_t stream, int sms) {
    const VLayout L = vlayout<NRT, NTILE, NMAT>(a.K, a.G, FMT, a.B);
    const void* fn = reinterpret_cast<const void*>(vp_gemv_kernel<FMT, NRT, NTILE, NMAT>);
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
    if (err != cudaSuccess) return err;
    const int items = a.max_groups * (a.R / (16 * NRT));
    const int grid = items < sms ? (items > 0 ? items : 1) : sms;
    VpArgs copy = a;
    void* args[] = {&copy};
    return launch_pdl_raw(fn, dim3(grid), dim3((vp_cw(FMT) + 1) * 32), L.total, stream, args);
}

}  // namespace

// Variants: gate/up (two matrices) and down (one matrix); items of the larger row block where
// shared memory allows; token groups of two tiles (8 tokens), or one tile (4 tokens) where no
// row block fits with two.
// row tiles per item: the larger (big) where shared memory allows, else the smaller
template <int FMT, int NMAT>
struct VpNrt {
    static constexpr int big = NMAT == 2 ? (FMT == DPA_FMT_UNIFORM ? kGuNRTUniform : kGuNRTBcq) : kDnNRT;
    static constexpr int small = NMAT == 2 ? kGuNRTSmall : kDnNRTSmall;
};

template <int FMT, int NMAT>
static size_t vp_bytes_f(bool big, int tpg, int K, int G, int B) {
    constexpr int NB = VpNrt<FMT, NMAT>::big, NS = VpNrt<FMT, NMAT>::small;
    if (big) return tpg == 2 ? vlayout<NB, 2, NMAT>(K, G, FMT, B).total : vlayout<NB, 1, NMAT>(K, G, FMT, B).total;
    return tpg == 2 ? vlayout<NS, 2, NMAT>(K, G, FMT, B).total : vlayout<NS, 1, NMAT>(K, G, FMT, B).total;
}
template <int NMAT>
static size_t vp_bytes(bool big, int tpg, int K, int G, int fmt, int B) {
    return fmt == DPA_FMT_UNIFORM ? vp_bytes_f<DPA_FMT_UNIFORM, NMAT>(big, tpg, K, G, B)
                                  : vp_bytes_f<DPA_FMT_BCQ, NMAT>(big, tpg, K, G, B);
}

int vp_tiles_per_group(int K_gateup, int K_down, int G, int fmt, int B) {
    const bool two = vp_bytes<2>(false, 2, K_gateup, G, fmt, B) <= kVpMaxSmem &&
                     vp_bytes<1>(false, 2, K_down, G, fmt, B) <= kVpMaxSmem;
    return two ? 2 : 1;
}

// the smallest configuration of a variant (the shape is supported when it fits)
size_t vp_smem_bytes(int K, int G, int fmt, int B, int nmat, int tiles_per_group) {
    return nmat == 2 ? vp_bytes<2>(false, tiles_per_group, K, G, fmt, B)
                     : vp_bytes<1>(false, tiles_per_group, K, G, fmt, B);
}

template <int FMT, int NMAT>
static cudaError_t launch_kind(const VpArgs& a, cudaStream_t stream, int sms) {
    constexpr int NB = VpNrt<FMT, NMAT>::big, NS = VpNrt<FMT, NMAT>::small;
    const bool two = a.tiles_per_group == 2;
    const bool big = a.R % (16 * NB) == 0 && vp_bytes<NMAT>(true, two ? 2 : 1, a.K, a.G, FMT, a.B) <= kVpMaxSmem;
    if (big) return two ? launch_variant<FMT, NB, 2, NMAT>(a, stream, sms) : launch_variant<FMT, NB, 1, NMAT>(a, stream, sms);
    return two ? launch_variant<FMT, NS, 2, NMAT>(a, stream, sms) : launch_variant<FMT, NS, 1, NMAT>(a, stream, sms);
}

template <int FMT, int NMAT>
static bool vp_big(const VpArgs& a) {
    constexpr int NB = VpNrt<FMT, NMAT>::big;
    return a.R % (16 * NB) == 0 && vp_bytes<NMAT>(true, a.tiles_per_group == 2 ? 2 : 1, a.K, a.G, FMT, a.B) <= kVpMaxSmem;
}

int vp_rows_per_item(const VpArgs& a) {
    const bool uni = a.fmt == DPA_FMT_UNIFORM;
    if (a.nmat == 2) {
        const bool big = uni ? vp_big<DPA_FMT_UNIFORM, 2>(a) : vp_big<DPA_FMT_BCQ, 2>(a);
        return 16 * (big ? (uni ? kGuNRTUniform : kGuNRTBcq) : kGuNRTSmall);
    }
    const bool big = uni ? vp_big<DPA_FMT_UNIFORM, 1>(a) : vp_big<DPA_FMT_BCQ, 1>(a);
    return 16 * (big ? kDnNRT : kDnNRTSmall);
}

int vp_grid(const VpArgs& a, int sms) {
    const int items = a.max_groups * (a.R / vp_rows_per_item(a));
    return items < sms ? (items > 0 ? items : 1) : sms;
}

cudaError_t launch_vp_gemv(const VpArgs& a, cudaStream_t stream, int sms) {
    if (a.nmat == 2)
        return a.fmt == DPA_FMT_UNIFORM ? launch_kind<DPA_FMT_UNIFORM, 2>(a, stream, sms)
                                        : launch_kind<DPA_FMT_BCQ, 2>(a, stream, sms);
    return a.fmt == DPA_FMT_UNIFORM ? launch_kind<DPA_FMT_UNIFORM, 1>(a, stream, sms)
                                    : launch_kind<DPA_FMT_BCQ, 1>(a, stream, sms);
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
