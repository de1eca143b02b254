// Prefill expert FFN on the fifth-generation tensor cores: grouped GEMMs with the variable-plane
// weights decoded into shared memory, tcgen05 MMAs accumulating in tensor memory (TMEM).
//
// What it computes (DPA-MoE / MatMoE pages, "Floor-and-Compensation"): for every token tile of one
// (expert e, plane count k) class,
//     gate/up:  a = W_gate^(k) x,  u = W_up^(k) x,  h = silu(a) * u          (h stored as fp16)
//     down:     o = W_down^(k) h                                              (fp32, per pair)
// with W^(k)[n, j] = s[n, g] * (q_hat^(k)[n, j] - z[n, g]) for j in group g, and
// q_hat^(k) = (q >> (B-k)) * 2^(B-k) + (2^(B-k) - 1) / 2.
//
// Exact operands, scale on the accumulator. z is an integer, so q_hat - z is a multiple of 1/2
// with |q_hat - z| < 2^B <= 16: exact in bf16 and fp16. The A operand (weights) is that value;
// the per-group scale s is applied when each group's fp32 accumulator is drained from TMEM,
// so the only roundings are the fp32 accumulation and, for the down GEMM, h rounded to fp16.
//
// Orientation: the MMA's M = 128 weight rows, N = the tile's tokens (padded to 16), K = 64 per
// pipeline stage (one 128-byte swizzle atom of 16-bit values). The weight row is the TMEM lane,
// so the group scale is a per-thread constant in the drain. Gate/up tiles hold 64 gate and the
// same 64 up rows, interleaved by 16 inside each 32-lane quadrant, so that SwiGLU pairs lane t
// with lane t ^ 16 of the same warp.
//
// Roles (576 threads, one CTA per SM, persistent over the work items (token tile, row block)):
//   warps 0-3   drain: tcgen05.ld each finished group's accumulator and the running sum,
//               run += s[n, g] * acc, tcgen05.st the running sum (TMEM columns 384..511);
//               epilogue per item (SwiGLU -> fp16 h, or fp32 per-pair outputs)
//   warps 4-15  decoders, three groups of four warps; group q fills A slot q (K stages
//               c = q mod 3): plane words of a stage -> swizzled K-major A tile; fence; arrive
//   warp 16     loader: TMA tensor loads, no multicast. Plane words: per (plane, matrix) one box
//               of 4 (gate/up) or 8 (down) row tiles x 4 stages of columns (a "plane stage"
//               holds 4 K stages). Activations: one 2D box of 128 rows x 64 columns per K stage
//               from the pair-ordered rows (x gathered by permute_rows_kernel, or h)
//   warp 17     TMEM allocation and the single MMA-issuing thread
// Every wait is bounded (globaltimer); on a timeout the kernel records DPA_ERR_DEVICE_TIMEOUT,
// every role leaves its loop, in-flight copies and MMAs are awaited, and TMEM is released.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kBM = 128;                  // weight rows per tile (MMA M)
constexpr int kBN = kGemmTileTokens;      // tokens per tile (MMA N <= 128)
constexpr int kBK = 64;                   // K per stage
constexpr int kAStages = 3;               // decoded weight tiles (MMA A operand)
constexpr int kLStages = 2 * kAStages;    // activation tiles (MMA B operand); one "chunk done" ring
                                          // of this depth frees both an A slot and a B slot
constexpr int kPStages = 3;               // plane stages
constexpr int kSC = 4;                    // K stages per plane stage
constexpr int kMaxPlanes = 4;
constexpr int kDecGroups = kAStages;       // decoder group q fills A slot q: chunks c = q (mod 3)
constexpr int kDecWarps = 4;                // warps per decoder group
constexpr int kThreads = (4 + kDecGroups * kDecWarps + 2) * 32;   // 576
constexpr int kLoaderWarp = 4 + kDecGroups * kDecWarps, kMmaWarp = kLoaderWarp + 1;
constexpr int kAccBufs = 3;               // group accumulators at TMEM columns 0, 128, 256
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kRunCol = 384;         // running sum of the scaled groups

constexpr int kATile = kBM * 128;                       // 16 KB
constexpr int kBTile = kBN * 128;                       // 16 KB
constexpr int kPlaneStage = kMaxPlanes * 8 * kSC * 128;   // 16 KB

struct GemmSmem {
    static constexpr int a = 0;
    static constexpr int b = a + kAStages * kATile;
    static constexpr int planes = b + kLStages * kBTile;
    // epilogue transposes, per drain warp: [32 tokens][16 rows] fp16 (gate/up) or [32][32] fp32 (down)
    static constexpr int epi = planes + kPStages * kPlaneStage;
    static constexpr int epi_warp = 32 * 33 * 4;   // fp32 rows padded to 33 words (bank-conflict free)
    // loaded[L], cdone[L], loadedP[P], emptyP[P], full[A], acc_full[3], acc_empty[3], done
    static constexpr int bars = epi + 4 * epi_warp;
    static constexpr int nbars = 2 * kLStages + 2 * kPStages + kAStages + 2 * kAccBufs + 1;
    static constexpr int misc = bars + nbars * 8;   // tmem address, abort flag
    static constexpr int total = misc + 16;
};
static_assert(GemmSmem::total + 1024 <= 232448, "stage rings exceed the shared memory of one CTA");

// ---- tcgen05 wrappers (inline PTX) ----
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);          // start address
    d |= static_cast<uint64_t>(1) << 16;                        // leading byte offset (unused with swizzle)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;                // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                        // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                        // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, A and B both bf16 (fmt 1) or fp16 (0),
// both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t instr_desc(int fmt, int n) {
    return (1u << 4) | (static_cast<uint32_t>(fmt) << 7) | (static_cast<uint32_t>(fmt) << 10) |
           (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(kBM >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

#define DPA_R32(r) \
    "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), \
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), \
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), \
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define DPA_W32(r)                                                                                                 \
    "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), \
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),          \
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),          \
        "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])

// 32 lanes x 32 consecutive 32-bit columns: thread t receives lane (base lane + t). Completes at
// tmem_wait_ld().
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : DPA_R32(r)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        DPA_W32(r)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- bulk and tensor copies into shared memory (no multicast) ----
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Four rows (r0..r3) of 64 consecutive 16-bit values starting at column x, 128-byte swizzled.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, int x, int r0, int r1, int r2, int r3,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
        : "memory");
}

// One box (64 columns x the map's box rows) at (x, y), 128-byte swizzled.
__device__ __forceinline__ void tma_tile2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_tile4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                           uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_tile5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3, int c4,
                                           uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar))
        : "memory");
}

// true in exactly one lane of the (fully active) warp
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Packed 16-bit subtraction a - b on both halves (bf16x2 or f16x2); exact here (see top).
template <bool F16>
__device__ __forceinline__ uint32_t sub2(uint32_t a, uint32_t b) {
    uint32_t r;
    if constexpr (F16) asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    else asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Both halves = v (a multiple of 1/4 in [32, 128), exact in bf16 and fp16).
template <bool F16>
__device__ __forceinline__ uint32_t half2_of(float v) {
    uint32_t u;
    if constexpr (F16) u = __half_as_ushort(__float2half_rn(v));
    else u = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    return u | (u << 16);
}

struct Item {
    int e, k, pos0, n, rb;
};

__device__ __forceinline__ Item load_item(const GemmArgs& a, int it, int RB) {
    const int tile = it / RB;
    const int4 t = __ldg(a.gtiles + tile);
    Item r;
    r.e = t.x;
    r.k = t.y;
    r.pos0 = t.z;
    r.n = t.w;
    r.rb = it - tile * RB;
    return r;
}

// Matrix and matrix row of A-tile row R (0..127) of row block rb.
template <bool DOWN>
__device__ __forceinline__ void a_row(int R, int rb, int& m, int& row) {
    if constexpr (DOWN) {
        m = 2;
        row = rb * kBM + R;
    } else {
        const int q = R >> 5, t = R & 31;
        m = t >> 4;
        row = rb * 64 + q * 16 + (t & 15);
    }
}

// Matrix and matrix row tile (16 rows) of A-tile row tile i (0..7).
template <bool DOWN>
__device__ __forceinline__ void a_rowtile(int i, int rb, int& m, int& rt) {
    if constexpr (DOWN) {
        m = 2;
        rt = rb * 8 + i;
    } else {
        m = i & 1;
        rt = rb * 4 + (i >> 1);
    }
}

struct Geo {
    int Kdim, RB, nchunks, ng, nblk, G;
    uint64_t plane_bytes;   // one plane of one matrix
};

template <bool DOWN>
__device__ __forceinline__ Geo make_geo(const GemmArgs& a) {
    Geo g;
    g.Kdim = DOWN ? a.I : a.H;
    g.RB = DOWN ? a.H / kBM : a.I / 64;
    g.nchunks = g.Kdim / kBK;
    g.G = a.G;
    g.ng = g.Kdim / a.G;
    g.nblk = g.Kdim / 64;
    g.plane_bytes = static_cast<uint64_t>(a.H) * a.I / 8;
    return g;
}

// ---- decoder: plane words of one stage -> A tile ----
// Thread p covers A row tile i = p >> 5 and lane l = p & 31 (g = l >> 2, c = l & 3) of the stage's
// 64-column block: rows g and g+8, columns 32*m_lo + 16*rho_hi + 4c + [0, 4) for each (rho, m_lo):
// eight 8-byte pieces.
// Plane stage layout: gate/up [plane][matrix][4 row tiles][kSC x 128 bytes],
// down [plane][8 row tiles][kSC x 128 bytes]; A row tile i is (row tile i >> 1, matrix i & 1) for
// gate/up and row tile i for down.
template <bool DOWN>
__device__ __forceinline__ int plane_off(int pl, int i) {
    if constexpr (DOWN) return (pl * 8 + i) * (kSC * 128);
    else return ((pl * 2 + (i & 1)) * 4 + (i >> 1)) * (kSC * 128);
}

// Thread p (0..127 of a decoder group) covers A row tile i = p >> 4 and lanes 2w, 2w+1
// (w = p & 15; g = w >> 1, c = 2 (w & 1) + {0, 1}) of the stage's 64-column block: rows g and g+8,
// columns 32*m_lo + 16*rho_hi + 8*(w & 1) + [0, 8) for each (rho, m_lo): eight 16-byte chunks.
template <bool DOWN, int B>
__device__ __forceinline__ void decode_stage(const unsigned char* sp, unsigned char* sa, int k, uint32_t K0,
                                             uint32_t K1, int p) {   // sp: this K stage's 128-byte column
    const int i = p >> 4, w = p & 15, g8 = w >> 1, hsel = w & 1;
    uint32_t wx[kMaxPlanes], wy[kMaxPlanes];
#pragma unroll
    for (int pl = 0; pl < B; ++pl) {
        if (pl < k) {
            const uint2 v = *reinterpret_cast<const uint2*>(sp + plane_off<DOWN>(pl, i) + (2 * w) * 4);
            wx[pl] = v.x;
            wy[pl] = v.y;
        } else {
            wx[pl] = 0u;
            wy[pl] = 0u;
        }
    }
    const int R0 = 16 * i + g8, R1 = R0 + 8;
#pragma unroll
    for (int rho = 0; rho < 4; ++rho) {
        // nibble m of N0 / N1 = the code (plane 0 = MSB) at position rho of lanes 2w / 2w+1: in
        // plane pl that bit sits at 4m + (B-1-pl) - rho (mod 32), so the planes merge under fixed
        // masks and one rotation by rho puts every nibble in place (planes >= k read as zero)
        uint32_t N0 = wx[0], N1 = wy[0];
#pragma unroll
        for (int pl = 1; pl < B; ++pl) {
            const uint32_t M = 0x11111111u << ((B - 1 - pl - rho) & 3);
            N0 = (N0 & ~M) | (wx[pl] & M);
            N1 = (N1 & ~M) | (wy[pl] & M);
        }
        N0 = __funnelshift_l(N0, N0, rho);
        N1 = __funnelshift_l(N1, N1, rho);
        const int R = (rho & 1) ? R1 : R0;
        const uint32_t Kr = (rho & 1) ? K1 : K0;
#pragma unroll
        for (int mlo = 0; mlo < 2; ++mlo) {
            uint32_t b0, b1, hi;
            if constexpr (DOWN) {   // fp16 64 + c: high byte 0x54, low byte c << 4
                b0 = (mlo ? N0 : (N0 << 4)) & 0xF0F0F0F0u;
                b1 = (mlo ? N1 : (N1 << 4)) & 0xF0F0F0F0u;
                hi = 0x54u;
            } else {                // bf16 64 + c: high byte 0x42, low byte 0x80 | (c << 1)
                b0 = ((mlo ? (N0 >> 3) : (N0 << 1)) & 0x1E1E1E1Eu) | 0x80808080u;
                b1 = ((mlo ? (N1 >> 3) : (N1 << 1)) & 0x1E1E1E1Eu) | 0x80808080u;
                hi = 0x42u;
            }
            uint4 v;
            v.x = sub2<DOWN>(prmt(b0, hi, 0x4140u), Kr);
            v.y = sub2<DOWN>(prmt(b0, hi, 0x4342u), Kr);
            v.z = sub2<DOWN>(prmt(b1, hi, 0x4140u), Kr);
            v.w = sub2<DOWN>(prmt(b1, hi, 0x4342u), Kr);
            const int chunk = 4 * mlo + 2 * (rho >> 1) + hsel;
            *reinterpret_cast<uint4*>(sa + R * 128 + ((chunk ^ (R & 7)) << 4)) = v;
        }
    }
}

__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.f + __expf(-v)); }

template <bool DOWN, int B>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(GemmArgs a, const __grid_constant__ CUtensorMap tmap,
                                                              const __grid_constant__ CUtensorMap pmap) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + GemmSmem::bars);
    uint64_t* loaded = bars;                         // [kLStages] copies of a stage landed
    uint64_t* cdone = loaded + kLStages;             // [kLStages] MMAs of chunk c done (slot c % kLStages)
    uint64_t* loadedP = cdone + kLStages;            // [kPStages] plane words of a plane stage landed
    uint64_t* emptyP = loadedP + kPStages;           // [kPStages] decoders done with a plane stage
    uint64_t* full = emptyP + kPStages;              // [kAStages] decoded A ready
    uint64_t* acc_full = full + kAStages;            // [kAccBufs]
    uint64_t* acc_empty = acc_full + kAccBufs;       // [kAccBufs]
    uint64_t* done = acc_empty + kAccBufs;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(sm + GemmSmem::misc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + GemmSmem::misc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < kLStages; ++i) {
            mbar_init(&loaded[i], 1);
            mbar_init(&cdone[i], 1);
        }
        // consumer barriers count one arrival per warp (lane 0 after __syncwarp), not per thread
        for (int i = 0; i < kPStages; ++i) {
            mbar_init(&loadedP[i], 1);
            mbar_init(&emptyP[i], kSC * kDecWarps);   // each of its kSC stages, by one group's warps
        }
        for (int i = 0; i < kAStages; ++i) {
            mbar_init(&full[i], kDecWarps);
        }
        for (int i = 0; i < kAccBufs; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(done, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(const_cast<uint32_t*>(s_tmem))),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    pdl_wait();   // tiles, positions and (down) h come from the previous kernels
    const Geo geo = make_geo<DOWN>(a);
    const int n_items = static_cast<int>(__ldcg(&a.hdr->n_gtiles)) * geo.RB;
    const int n_mine = n_items > static_cast<int>(blockIdx.x)
                           ? (n_items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;

    if (warp == kLoaderWarp) {
        // ================= loader: one lane issues every tensor load =================
        if (lane == 0) {
            int c = 0, cp = 0;
            bool ok = true;
            for (int j = 0; j < n_mine && ok; ++j) {
                const Item it = load_item(a, static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x), geo.RB);
                const uint32_t pbytes = static_cast<uint32_t>(it.k) * 8 * kSC * 128;
                for (int kc = 0; kc < geo.nchunks; ++kc, ++c) {
                    if (kc % kSC == 0) {   // next plane stage: k planes x (2 matrices | 1) boxes
                        const int ps = cp % kPStages, pr = cp / kPStages;
                        if (*s_abort || !mbar_wait_bounded(&emptyP[ps], (pr & 1) ^ 1, a.hdr, 0x613)) {
                            *s_abort = 1;
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&loadedP[ps], pbytes);
                        unsigned char* sp = sm + GemmSmem::planes + ps * kPlaneStage;
                        for (int pl = 0; pl < it.k; ++pl) {
                            if constexpr (DOWN) {
                                tma_tile4d(sp + plane_off<DOWN>(pl, 0), &pmap, kc * 32, it.rb * 8, pl, it.e, &loadedP[ps]);
                            } else {
                                tma_tile5d(sp + plane_off<DOWN>(pl, 0), &pmap, kc * 32, it.rb * 4, pl, 0, it.e,
                                           &loadedP[ps]);
                                tma_tile5d(sp + plane_off<DOWN>(pl, 1), &pmap, kc * 32, it.rb * 4, pl, 1, it.e,
                                           &loadedP[ps]);
                            }
                        }
                        ++cp;
                    }
                    const int s = c % kLStages, r = c / kLStages;
                    if (*s_abort || !mbar_wait_bounded(&cdone[s], (r & 1) ^ 1, a.hdr, 0x610)) {
                        *s_abort = 1;
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&loaded[s], static_cast<uint32_t>(kBTile));
                    tma_tile2d(sm + GemmSmem::b + s * kBTile, &tmap, kc * kBK, it.pos0, &loaded[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4 && warp < kLoaderWarp) {
        // ================= decoders: group q decodes chunks q, q+3, ... into A slot q =================
        const int q = (warp - 4) / kDecWarps;
        const int p = tid - 128 - q * kDecWarps * 32;
        const int i = p >> 4, g8 = (p & 15) >> 1;
        const int gshift = 31 - __clz(geo.G / kBK);   // K stages per scale group is a power of two
        int j = 0, kc = q, jcur = -1, rq = 0;
        bool ok = true;
        Item it{};
        const uint32_t* mrow0 = nullptr;
        const uint32_t* mrow1 = nullptr;
        float d = 0.f;
        for (int c = q; j < n_mine && ok; c += kDecGroups, ++rq) {
            if (j != jcur) {
                it = load_item(a, static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x), geo.RB);
                int m0, r0, m1, r1;
                a_row<DOWN>(16 * i + g8, it.rb, m0, r0);
                a_row<DOWN>(16 * i + g8 + 8, it.rb, m1, r1);
                const uint8_t* mb = a.meta + static_cast<uint64_t>(it.e) * a.meta_per_expert;
                mrow0 = reinterpret_cast<const uint32_t*>(mb + a.meta_mat_off[m0]) + static_cast<uint64_t>(r0) * geo.ng;
                mrow1 = reinterpret_cast<const uint32_t*>(mb + a.meta_mat_off[m1]) + static_cast<uint64_t>(r1) * geo.ng;
                d = 0.5f * static_cast<float>((1 << (B - it.k)) - 1);
                jcur = j;
            }
            // zeros of this thread's two rows for this stage's group (latency overlaps the waits)
            const uint32_t zz0 = __ldg(mrow0 + (kc >> gshift)), zz1 = __ldg(mrow1 + (kc >> gshift));
            const int cpi = c / kSC, ps = cpi % kPStages;
            // A slot q was last read by the MMAs of chunk c - kAStages
            const int cprev = c - kAStages;
            const bool w_ok = !*s_abort && mbar_wait_bounded(&loadedP[ps], (cpi / kPStages) & 1, a.hdr, 0x611) &&
                              (cprev < 0 ||
                               mbar_wait_bounded(&cdone[cprev % kLStages], (cprev / kLStages) & 1, a.hdr, 0x612));
            if (!__all_sync(0xffffffffu, w_ok)) {   // the warp leaves together (it synchronises below)
                *s_abort = 1;
                ok = false;
                break;
            }
            // constants 64 - (d - z): subtracted from 64 + c'' they leave q_hat - z
            const uint32_t K0 = half2_of<DOWN>(64.f - (d - __half2float(__ushort_as_half(static_cast<unsigned short>(zz0 >> 16)))));
            const uint32_t K1 = half2_of<DOWN>(64.f - (d - __half2float(__ushort_as_half(static_cast<unsigned short>(zz1 >> 16)))));
            decode_stage<DOWN, B>(sm + GemmSmem::planes + ps * kPlaneStage + (c % kSC) * 128,
                                  sm + GemmSmem::a + q * kATile, it.k, K0, K1, p);
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                mbarrier_arrive(&full[q]);
                mbarrier_arrive(&emptyP[ps]);   // this stage's slice of the plane stage is consumed
            }
            kc += kDecGroups;
            if (kc >= geo.nchunks) {
                kc -= geo.nchunks;
                ++j;
            }
        }
    } else if (warp == kMmaWarp) {
        // ================= MMA issue (one elected thread) =================
        // The whole warp runs this loop in uniform control flow (so the descriptors and ring
        // counters stay in uniform registers) and one elected lane issues each tcgen05 operation.
        // Ring indices are counters; descriptors are precomputed per slot and advanced by 32
        // bytes (+2) per MMA.
        const bool leader = elect_one();
        const uint32_t fmt = DOWN ? 0u : 1u;
        const uint32_t a_base = smem_u32(sm + GemmSmem::a), b_base = smem_u32(sm + GemmSmem::b);
        const uint64_t dconst = smem_desc_sw128(0);
        const int cpg = geo.G / kBK;   // K stages per scale group
        int s = 0, rs = 0, sa = 0, ra = 0, gb = 0, gr = 0;   // gb, gr: accumulator buffer, round
        bool ok = true;
        for (int j = 0; j < n_mine && ok; ++j) {
            const Item item = load_item(a, static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x), geo.RB);
            const uint32_t idesc = instr_desc(static_cast<int>(fmt), (item.n + 15) & ~15);
            int kin = 0;
            for (int kc = 0; kc < geo.nchunks; ++kc) {
                const bool first = kin == 0, last = kin == cpg - 1;
                const int b = gb;
                bool w_ok = !first || mbar_wait_bounded(&acc_empty[b], (gr & 1) ^ 1, a.hdr, 0x620);
                w_ok = w_ok && mbar_wait_bounded(&loaded[s], rs & 1, a.hdr, 0x623) &&
                       mbar_wait_bounded(&full[sa], ra & 1, a.hdr, 0x621);
                if (!__all_sync(0xffffffffu, w_ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = dconst | ((a_base + static_cast<uint32_t>(sa) * kATile) >> 4);
                const uint64_t bd = dconst | ((b_base + static_cast<uint32_t>(s) * kBTile) >> 4);
                const uint32_t td = tmem + static_cast<uint32_t>(b) * kBN;
                if (leader) {
                    tc_mma(td, ad, bd, idesc, first ? 0u : 1u);
                    tc_mma(td, ad + 2, bd + 2, idesc, 1u);
                    tc_mma(td, ad + 4, bd + 4, idesc, 1u);
                    tc_mma(td, ad + 6, bd + 6, idesc, 1u);
                    tc_commit(&cdone[s]);
                    if (last) tc_commit(&acc_full[b]);
                }
                __syncwarp();
                if (last && ++gb == kAccBufs) { gb = 0; ++gr; }
                kin = last ? 0 : kin + 1;
                if (++s == kLStages) { s = 0; ++rs; }
                if (++sa == kAStages) { sa = 0; ++ra; }
            }
            if (*s_abort) ok = false;
        }
        if (!ok) *s_abort = 1;
        // every MMA issued has completed before TMEM is released
        if (leader) tc_commit(done);
        __syncwarp();
        mbar_wait_bounded(done, 0, a.hdr, 0x622);
        __syncwarp();
    } else {
        // ================= drain + epilogue (warps 0-3, TMEM lanes 32*warp ...) =================
        const int R = 32 * warp + lane;
        const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
        int gb = 0, gr = 0;   // accumulator buffer and its round
        bool ok = true;
        for (int j = 0; j < n_mine && ok; ++j) {
            const Item item = load_item(a, static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x), geo.RB);
            int m, row;
            a_row<DOWN>(R, item.rb, m, row);
            const uint32_t* mrow = reinterpret_cast<const uint32_t*>(
                a.meta + static_cast<uint64_t>(item.e) * a.meta_per_expert + a.meta_mat_off[m] +
                static_cast<uint64_t>(row) * geo.ng * 4);
            const int nch = (item.n + 31) >> 5;
            uint32_t sz_next = __ldg(mrow);
            for (int g = 0; g < geo.ng; ++g) {
                const float sc = __half2float(__ushort_as_half(static_cast<unsigned short>(sz_next & 0xFFFF)));
                if (g + 1 < geo.ng) sz_next = __ldg(mrow + g + 1);
                const int b = gb;
                const bool w_ok = !*s_abort && mbar_wait_bounded(&acc_full[b], gr & 1, a.hdr, 0x630);
                if (!__all_sync(0xffffffffu, w_ok)) {   // warp-uniform: tcgen05.ld below is .sync.aligned
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int q = 0; q < nch; ++q) {   // warp-uniform
                    uint32_t v[32], run[32];
                    tmem_ld32(tmem + lane_base + b * kBN + 32 * q, v);
                    if (g > 0) tmem_ld32(tmem + lane_base + kRunCol + 32 * q, run);
                    tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const float acc = g > 0 ? __uint_as_float(run[u]) : 0.f;
                        run[u] = __float_as_uint(fmaf(sc, __uint_as_float(v[u]), acc));
                    }
                    tmem_st32(tmem + lane_base + kRunCol + 32 * q, run);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbarrier_arrive(&acc_empty[b]);
                if (++gb == kAccBufs) { gb = 0; ++gr; }
            }
            if (!ok) break;
            if constexpr (DOWN) {
                // transpose 32 tokens x this warp's 32 rows through shared memory; each lane then
                // stores the 32 rows of one token as eight 16-byte pieces
                float* out0 = a.out_pair + static_cast<uint64_t>(item.pos0) * a.H + (row - lane);
                float* st = reinterpret_cast<float*>(sm + GemmSmem::epi + warp * GemmSmem::epi_warp);
                for (int q = 0; q < nch; ++q) {
                    uint32_t run[32];
                    tmem_ld32(tmem + lane_base + kRunCol + 32 * q, run);
                    tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 32; ++u) st[u * 33 + lane] = __uint_as_float(run[u]);   // padded rows
                    __syncwarp();
                    const int tok = 32 * q + lane;
                    if (tok < item.n) {
                        float4* dst = reinterpret_cast<float4*>(out0 + static_cast<uint64_t>(tok) * a.H);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            __stcs(dst + v, make_float4(st[lane * 33 + 4 * v], st[lane * 33 + 4 * v + 1],
                                                        st[lane * 33 + 4 * v + 2], st[lane * 33 + 4 * v + 3]));
                    }
                    __syncwarp();
                }
            } else {
                // lanes t < 16 hold gate rows, t >= 16 the up rows of the same outputs. For each token
                // pair (2u, 2u+1) one exchange gives the gate lane the up value of token 2u and the up
                // lane the gate value of token 2u+1; every lane then finishes one token. All 16
                // values of a 32-token chunk are computed before any store (independent chains).
                const bool is_gate = (lane & 16) == 0;
                // h rows n0 + 16 * warp + [0, 16) of this warp's quadrant (row of lane 0)
                __half* hb0 = reinterpret_cast<__half*>(a.hbuf) + static_cast<uint64_t>(item.pos0) * a.I +
                              (row - (lane & 15));
                bool overflow = false;
                for (int q = 0; q < nch; ++q) {
                    uint32_t run[32];
                    tmem_ld32(tmem + lane_base + kRunCol + 32 * q, run);
                    tmem_wait_ld();
                    float hv[16];
#pragma unroll
                    for (int u2 = 0; u2 < 16; ++u2) {
                        const float ev = __uint_as_float(run[2 * u2]), od = __uint_as_float(run[2 * u2 + 1]);
                        const float recv = __shfl_xor_sync(0xffffffffu, is_gate ? od : ev, 16);
                        const float gv = is_gate ? ev : recv, uv = is_gate ? recv : od;
                        hv[u2] = silu_f(gv) * uv;
                    }
                    // transpose through shared memory: [token][16 rows] fp16, then each lane stores
                    // 8 rows of one token (16 bytes) per instruction
                    __half* st = reinterpret_cast<__half*>(sm + GemmSmem::epi + warp * GemmSmem::epi_warp);
                    const int r16 = lane & 15, par = is_gate ? 0 : 1;
#pragma unroll
                    for (int u2 = 0; u2 < 16; ++u2) {
                        overflow |= (32 * q + 2 * u2 + par < item.n) && !(fabsf(hv[u2]) <= 65504.f);
                        st[(2 * u2 + par) * 16 + r16] = __float2half_rn(hv[u2]);
                    }
                    __syncwarp();
                    const int tok = 32 * q + lane;
                    if (tok < item.n) {
                        const uint4* src = reinterpret_cast<const uint4*>(st + lane * 16);
                        uint4* dst = reinterpret_cast<uint4*>(hb0 + static_cast<uint64_t>(tok) * a.I);
                        dst[0] = src[0];
                        dst[1] = src[1];
                    }
                    __syncwarp();
                }
                if (overflow) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 0x640);
            }
        }
        if (!ok) *s_abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ---- host: tensor maps for the activation operand ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// rows x cols row-major 16-bit matrix, boxes of 64 columns x box_rows, 128-byte swizzle, zero fill
bool make_map(CUtensorMap* map, const void* base, bool f16, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t gemm_tc_smem_bytes() { return GemmSmem::total + 1024; }

// Plane words as a u32 tensor: gate/up {row-tile words (H/2), row tiles (I/16), planes, matrix
// (gate, up), experts}; down {row-tile words (I/2), row tiles (H/16), planes, experts}. Boxes of
// kSC column blocks (kSC x 32 words) x 4 (gate/up) or 8 (down) row tiles, no swizzle.
bool make_plane_map(CUtensorMap* map, const GemmArgs& a, bool down) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint64_t plane = static_cast<uint64_t>(a.H) * a.I / 8;
    const uint64_t rt_bytes = down ? static_cast<uint64_t>(a.I) * 2 : static_cast<uint64_t>(a.H) * 2;
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if (down) {
        const cuuint64_t dims[4] = {rt_bytes / 4, static_cast<uint64_t>(a.H) / 16, static_cast<uint64_t>(a.B),
                                    static_cast<uint64_t>(a.E)};
        const cuuint64_t strides[3] = {rt_bytes, plane, a.planes_per_expert};
        const cuuint32_t box[4] = {kSC * 32, 8, 1, 1};
        return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint8_t*>(a.planes + a.planes_mat_off[2]), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    const cuuint64_t dims[5] = {rt_bytes / 4, static_cast<uint64_t>(a.I) / 16, static_cast<uint64_t>(a.B), 2,
                                static_cast<uint64_t>(a.E)};
    const cuuint64_t strides[4] = {rt_bytes, plane, a.planes_mat_off[1], a.planes_per_expert};
    const cuuint32_t box[5] = {kSC * 32, 4, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 5, const_cast<uint8_t*>(a.planes + a.planes_mat_off[0]), dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool DOWN, int B>
static cudaError_t launch_one(const GemmArgs& a, const CUtensorMap& map, const CUtensorMap& pmap, cudaStream_t stream,
                              int sms) {
    const void* fn = reinterpret_cast<const void*>(gemm_tc_kernel<DOWN, B>);
    const size_t smem = gemm_tc_smem_bytes();
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    GemmArgs copy = a;
    alignas(64) CUtensorMap m = map;
    alignas(64) CUtensorMap pm = pmap;
    void* args[] = {&copy, &m, &pm};
    return launch_pdl_raw(fn, dim3(sms), dim3(kThreads), smem, stream, args);
}

template <bool DOWN>
static cudaError_t launch_b(const GemmArgs& a, cudaStream_t stream, int sms) {
    alignas(64) CUtensorMap map, pmap;
    // activations in grouped pair order: x gathered per pair (gate/up) or h (down), 128-row boxes
    const bool ok = (DOWN ? make_map(&map, a.hbuf, true, static_cast<uint64_t>(a.P), a.I, kBN)
                          : make_map(&map, a.xperm, false, static_cast<uint64_t>(a.P), a.H, kBN)) &&
                    make_plane_map(&pmap, a, DOWN);
    if (!ok) return cudaErrorInvalidValue;
    switch (a.B) {
        case 1: return launch_one<DOWN, 1>(a, map, pmap, stream, sms);
        case 2: return launch_one<DOWN, 2>(a, map, pmap, stream, sms);
        case 3: return launch_one<DOWN, 3>(a, map, pmap, stream, sms);
        case 4: return launch_one<DOWN, 4>(a, map, pmap, stream, sms);
        default: return cudaErrorInvalidValue;
    }
}

// x rows in grouped pair order: xperm[pos] = x[token of pos]; one warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint16_t* x, const int32_t* pos_tok, uint16_t* xperm,
                                                           int P, int H) {
    pdl_wait();
    const int pos = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (pos >= P) return;
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(__ldg(pos_tok + pos)) * H);
    uint4* dst = reinterpret_cast<uint4*>(xperm + static_cast<size_t>(pos) * H);
    for (int c = lane; c < H / 8; c += 32) dst[c] = __ldg(src + c);
}

cudaError_t launch_permute_rows(const GemmArgs& a, cudaStream_t stream) {
    GemmArgs b = a;
    const uint16_t* x = b.x;
    const int32_t* pt = b.pos_tok;
    uint16_t* xp = b.xperm;
    int P = b.P, H = b.H;
    void* args[] = {&x, &pt, &xp, &P, &H};
    return launch_pdl_raw(reinterpret_cast<const void*>(permute_rows_kernel), dim3((P + 7) / 8), dim3(256), 0, stream,
                          args);
}

cudaError_t launch_gemm_gateup(const GemmArgs& a, cudaStream_t stream, int sms) { return launch_b<false>(a, stream, sms); }
cudaError_t launch_gemm_down(const GemmArgs& a, cudaStream_t stream, int sms) { return launch_b<true>(a, stream, sms); }

}  // namespace dpa
