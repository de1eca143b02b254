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
// Roles (288 threads, one CTA per SM, persistent over the work items (token tile, row block)):
//   warps 0-3  drain: tcgen05.ld each finished group's accumulator, run += s[n, g] * acc in
//              registers, then the epilogue (SwiGLU -> fp16 h, or fp32 per-pair outputs)
//   warps 4-7  producers: cp.async of plane words, scales/zeros and activation rows into the
//              stage ring; decode the planes into the swizzled K-major A tile; fence; arrive
//   warp 8     TMEM allocation and the single MMA-issuing thread
// Every wait is bounded (globaltimer); on a timeout the kernel records DPA_ERR_DEVICE_TIMEOUT,
// every role leaves its loop, in-flight copies and MMAs are awaited, and TMEM is released.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kBM = 128;                  // weight rows per tile (MMA M)
constexpr int kBN = kGemmTileTokens;      // tokens per tile (MMA N <= 128)
constexpr int kBK = 64;                   // K per stage
constexpr int kStages = 6;
constexpr int kMaxPlanes = 4;
constexpr int kLookahead = 2;             // producer: stages loaded ahead of the one being decoded
constexpr int kThreads = 288;
constexpr int kProdThreads = 128;
constexpr uint32_t kTmemCols = 512;       // two 128-column accumulators (power of two >= 32)

constexpr int kATile = kBM * 128;                       // 16 KB
constexpr int kBTile = kBN * 128;                       // 16 KB
constexpr int kPlaneStage = kMaxPlanes * 8 * 128;       // 4 KB
constexpr int kMetaStage = kBM * 4;                     // 512 B

struct GemmSmem {
    static constexpr int a = 0;
    static constexpr int b = a + kStages * kATile;
    static constexpr int planes = b + kStages * kBTile;
    static constexpr int meta = planes + kStages * kPlaneStage;
    static constexpr int bars = meta + kStages * kMetaStage;   // full[S], empty[S], acc_full[2], acc_empty[2], done
    static constexpr int nbars = 2 * kStages + 5;
    static constexpr int misc = bars + nbars * 8;                // tmem address, abort flag
    static constexpr int total = misc + 16;
};
static_assert(GemmSmem::total + 1024 <= 232448, "stage ring exceeds the shared memory of one CTA");

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

// 32 lanes x 32 consecutive fp32 columns: thread t receives lane (base lane + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---- cp.async (Ampere-style, generic proxy) ----
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void producer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kProdThreads) : "memory"); }

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

// 16-bit encoding of 64 + c for a code c in [0, 16) (byte b holds the code, see decode_stage)
// and of a value v that is a multiple of 1/4 in [32, 128).
template <bool F16>
__device__ __forceinline__ uint32_t half2_of(float v) {
    if constexpr (F16) {
        const __half h = __float2half_rn(v);
        const uint32_t u = __half_as_ushort(h);
        return u | (u << 16);
    } else {
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        const uint32_t u = __bfloat16_as_ushort(h);
        return u | (u << 16);
    }
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
    int Kdim, Rows, RB, nchunks, ng, nblk, G, B;
    uint64_t plane_bytes;   // one plane of one matrix
};

template <bool DOWN>
__device__ __forceinline__ Geo make_geo(const GemmArgs& a) {
    Geo g;
    g.Kdim = DOWN ? a.I : a.H;
    g.Rows = DOWN ? a.H : a.I;
    g.RB = DOWN ? a.H / kBM : a.I / 64;
    g.nchunks = g.Kdim / kBK;
    g.G = a.G;
    g.ng = g.Kdim / a.G;
    g.nblk = g.Kdim / 64;
    g.B = a.B;
    g.plane_bytes = static_cast<uint64_t>(a.H) * a.I / 8;
    return g;
}

// ---- producer: issue the copies of one stage ----
template <bool DOWN>
__device__ __forceinline__ void issue_stage(const GemmArgs& a, const Geo& geo, const Item& it, int kc,
                                            unsigned char* sm, int s, int p, const int (&tok)[8]) {
    // plane words: k planes x 8 A row tiles x 128 bytes (lanes of one 64-column block)
    unsigned char* sp = sm + GemmSmem::planes + s * kPlaneStage;
    const uint8_t* pbase = a.planes + static_cast<uint64_t>(it.e) * a.planes_per_expert;
    for (int u = p; u < it.k * 64; u += kProdThreads) {
        const int pl = u >> 6, i = (u >> 3) & 7, piece = u & 7;
        int m, rt;
        a_rowtile<DOWN>(i, it.rb, m, rt);
        const uint8_t* src = pbase + a.planes_mat_off[m] + static_cast<uint64_t>(pl) * geo.plane_bytes +
                             (static_cast<uint64_t>(rt) * geo.nblk + kc) * 128 + piece * 16;
        cp_async16(sp + (pl * 8 + i) * 128 + piece * 16, src, 16);
    }
    // {s, z} of each A row for this stage's group
    {
        int m, row;
        a_row<DOWN>(p, it.rb, m, row);
        const int g = (kc * kBK) / geo.G;
        const uint8_t* src = a.meta + static_cast<uint64_t>(it.e) * a.meta_per_expert + a.meta_mat_off[m] +
                             (static_cast<uint64_t>(row) * geo.ng + g) * 4;
        cp_async4(sm + GemmSmem::meta + s * kMetaStage + p * 4, src);
    }
    // activation rows: row j, 16-byte chunk ch (= p & 7) into the swizzled K-major B tile
    unsigned char* sb = sm + GemmSmem::b + s * kBTile;
    const int n16 = (it.n + 15) & ~15;
    const int ch = p & 7;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int j = (p >> 3) + 16 * i;
        if (j < n16) {
            const uint16_t* src;
            if constexpr (DOWN)
                src = a.hbuf + static_cast<uint64_t>(it.pos0 + (j < it.n ? j : 0)) * a.I + kc * kBK + ch * 8;
            else
                src = a.x + static_cast<uint64_t>(tok[i]) * a.H + kc * kBK + ch * 8;
            cp_async16(sb + j * 128 + ((ch ^ (j & 7)) << 4), src, j < it.n ? 16u : 0u);
        }
    }
}

// ---- producer: decode the planes of one stage into the A tile ----
// Thread p covers A row tile i = p >> 4 and lanes 2w, 2w+1 (w = p & 15) of its 64-column block:
// rows g and g+8 (g = w >> 1), columns 16*rho_hi + 32*m_lo + 8*(w & 1) + [0, 8) for each
// (rho_hi, m_lo): eight 16-byte chunks.
template <bool DOWN, int B>
__device__ __forceinline__ void decode_stage(const Geo& geo, const Item& it, unsigned char* sm, int s, int p) {
    const int i = p >> 4, w = p & 15, g8 = w >> 1, hsel = w & 1;
    const unsigned char* sp = sm + GemmSmem::planes + s * kPlaneStage;
    uint32_t wx[kMaxPlanes], wy[kMaxPlanes];
#pragma unroll
    for (int pl = 0; pl < B; ++pl) {
        if (pl < it.k) {
            const uint2 v = *reinterpret_cast<const uint2*>(sp + (pl * 8 + i) * 128 + (2 * w) * 4);
            wx[pl] = v.x;
            wy[pl] = v.y;
        } else {
            wx[pl] = 0u;
            wy[pl] = 0u;
        }
    }
    // per-row constant 64 - (d - z), d = (2^(B-k) - 1) / 2: subtracting it from 64 + c'' leaves
    // c'' + d - z = q_hat - z
    const uint32_t* smeta = reinterpret_cast<const uint32_t*>(sm + GemmSmem::meta + s * kMetaStage);
    const float d = 0.5f * static_cast<float>((1 << (B - it.k)) - 1);
    const int R0 = 16 * i + g8, R1 = R0 + 8;
    const float z0 = __half2float(__ushort_as_half(static_cast<unsigned short>(smeta[R0] >> 16)));
    const float z1 = __half2float(__ushort_as_half(static_cast<unsigned short>(smeta[R1] >> 16)));
    const uint32_t K0 = half2_of<DOWN>(64.f - (d - z0));
    const uint32_t K1 = half2_of<DOWN>(64.f - (d - z1));
    unsigned char* sa = sm + GemmSmem::a + s * kATile;
#pragma unroll
    for (int rho = 0; rho < 4; ++rho) {
        // nibble m of N0 / N1 = code bits (plane 0 = MSB) at bit 4m + rho of lanes 2w / 2w+1
        uint32_t N0 = 0u, N1 = 0u;
#pragma unroll
        for (int pl = 0; pl < B; ++pl) {
            const int t = B - 1 - pl;
            N0 |= (t >= rho ? (wx[pl] << (t - rho)) : (wx[pl] >> (rho - t))) & (0x11111111u << t);
            N1 |= (t >= rho ? (wy[pl] << (t - rho)) : (wy[pl] >> (rho - t))) & (0x11111111u << t);
        }
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

__device__ __forceinline__ float silu_f(float v) { return v / (1.f + __expf(-v)); }

template <bool DOWN, int B>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(GemmArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + GemmSmem::bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* acc_full = bars + 2 * kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* done = acc_empty + 2;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(sm + GemmSmem::misc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + GemmSmem::misc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], kProdThreads);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 128);
        }
        mbar_init(done, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
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

    if (warp >= 4 && warp < 8) {
        // ================= producers =================
        const int p = tid - 128;
        const int n_mine = n_items > static_cast<int>(blockIdx.x)
                               ? (n_items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                               : 0;
        const int n_chunks = n_mine * geo.nchunks;
        int tok[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        Item cur{}, dec{};
        int dec_item = -1;
        bool ok = true;
        for (int c = 0; c < n_chunks + kLookahead; ++c) {
            if (c < n_chunks && ok) {
                const int s = c % kStages, r = c / kStages;
                const int j = c / geo.nchunks, kc = c - j * geo.nchunks;
                if (kc == 0) {
                    cur = load_item(a, static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x), geo.RB);
                    if constexpr (!DOWN) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int jj = (p >> 3) + 16 * i;
                            tok[i] = jj < cur.n ? __ldcg(a.pos_tok + cur.pos0 + jj) : 0;
                        }
                    }
                }
                if (*s_abort || !mbar_wait_bounded(&empty[s], (r & 1) ^ 1, a.hdr, 0x610)) {
                    *s_abort = 1;
                    ok = false;
                } else {
                    issue_stage<DOWN>(a, geo, cur, kc, sm, s, p, tok);
                }
            }
            cp_async_commit();   // (empty groups keep the wait_group arithmetic uniform)
            if (c >= kLookahead) {
                const int cd = c - kLookahead;
                cp_async_wait<kLookahead>();
                producer_sync();
                if (ok && cd < n_chunks && !*s_abort) {
                    const int j = cd / geo.nchunks;
                    if (j != dec_item) {
                        dec = load_item(a, static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x), geo.RB);
                        dec_item = j;
                    }
                    const int s = cd % kStages;
                    decode_stage<DOWN, B>(geo, dec, sm, s, p);
                    fence_proxy_async();
                    mbarrier_arrive(&full[s]);
                }
            }
        }
        cp_async_wait_all();
    } else if (warp == 8) {
        // ================= MMA issue (one thread) =================
        if (lane == 0) {
            const int fmt = DOWN ? 0 : 1;
            int c = 0, gc = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                const Item item = load_item(a, it, geo.RB);
                const uint32_t idesc = instr_desc(fmt, (item.n + 15) & ~15);
                for (int kc = 0; kc < geo.nchunks && ok; ++kc, ++c) {
                    const int s = c % kStages, r = c / kStages;
                    const bool first = (kc * kBK) % geo.G == 0;
                    const bool last = ((kc + 1) * kBK) % geo.G == 0;
                    const int b = gc & 1;
                    if (first && (*s_abort || !mbar_wait_bounded(&acc_empty[b], ((gc >> 1) & 1) ^ 1, a.hdr, 0x620))) {
                        ok = false;
                        break;
                    }
                    if (*s_abort || !mbar_wait_bounded(&full[s], r & 1, a.hdr, 0x621)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(sm + GemmSmem::a + s * kATile);
                    const uint32_t sb = smem_u32(sm + GemmSmem::b + s * kBTile);
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ++ks)
                        tc_mma(tmem + b * kBN, smem_desc_sw128(sa + ks * 32), smem_desc_sw128(sb + ks * 32), idesc,
                               (first && ks == 0) ? 0u : 1u);
                    tc_commit(&empty[s]);
                    if (last) {
                        tc_commit(&acc_full[b]);
                        ++gc;
                    }
                }
            }
            if (!ok) *s_abort = 1;
            // every MMA issued has completed before TMEM is released
            tc_commit(done);
            mbar_wait_bounded(done, 0, a.hdr, 0x622);
        }
        __syncwarp();
    } else {
        // ================= drain + epilogue (warps 0-3, TMEM lanes 32*warp ...) =================
        const int R = 32 * warp + lane;
        int gc = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const Item item = load_item(a, it, geo.RB);
            int m, row;
            a_row<DOWN>(R, item.rb, m, row);
            const uint32_t* mrow = reinterpret_cast<const uint32_t*>(
                a.meta + static_cast<uint64_t>(item.e) * a.meta_per_expert + a.meta_mat_off[m] +
                static_cast<uint64_t>(row) * geo.ng * 4);
            const int nch = (item.n + 31) >> 5;
            float run[kBN];
#pragma unroll
            for (int j = 0; j < kBN; ++j) run[j] = 0.f;
            uint32_t sz_next = __ldg(mrow);
            for (int g = 0; g < geo.ng; ++g, ++gc) {
                const float sc = __half2float(__ushort_as_half(static_cast<unsigned short>(sz_next & 0xFFFF)));
                if (g + 1 < geo.ng) sz_next = __ldg(mrow + g + 1);
                const int b = gc & 1;
                if (*s_abort || !mbar_wait_bounded(&acc_full[b], (gc >> 1) & 1, a.hdr, 0x630)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tb = tmem + (static_cast<uint32_t>(32 * warp) << 16) + b * kBN;
#pragma unroll
                for (int q = 0; q < kBN / 32; ++q) {
                    if (q < nch) {
                        float v[32];
                        tmem_ld32(tb + 32 * q, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) run[32 * q + i] = fmaf(sc, v[i], run[32 * q + i]);
                    }
                }
                tc_fence_before();
                mbarrier_arrive(&acc_empty[b]);
            }
            if (!ok) break;
            if constexpr (DOWN) {
                float* out = a.out_pair + static_cast<uint64_t>(item.pos0) * a.H + row;
#pragma unroll
                for (int j = 0; j < kBN; ++j)
                    if (j < item.n) __stcs(out + static_cast<uint64_t>(j) * a.H, run[j]);
            } else {
                // lanes t < 16 hold gate rows, t >= 16 the up rows of the same outputs; even
                // tokens are finished by the gate lane, odd ones by the up lane
                const bool is_gate = (lane & 16) == 0;
                __half* hb = reinterpret_cast<__half*>(a.hbuf) + static_cast<uint64_t>(item.pos0) * a.I + row;
                bool overflow = false;
#pragma unroll
                for (int j = 0; j < kBN; ++j) {
                    if (j < item.n) {   // warp-uniform
                        const float other = __shfl_xor_sync(0xffffffffu, run[j], 16);
                        if (is_gate == ((j & 1) == 0)) {
                            const float gv = is_gate ? run[j] : other, uv = is_gate ? other : run[j];
                            const float hv = silu_f(gv) * uv;
                            overflow |= !(fabsf(hv) <= 65504.f);
                            hb[static_cast<uint64_t>(j) * a.I] = __float2half_rn(hv);
                        }
                    }
                }
                if (overflow) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 0x640);
            }
        }
        if (!ok) *s_abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

}  // namespace

size_t gemm_tc_smem_bytes() { return GemmSmem::total + 1024; }

template <bool DOWN, int B>
static cudaError_t launch_one(const GemmArgs& a, cudaStream_t stream, int sms) {
    const void* fn = reinterpret_cast<const void*>(gemm_tc_kernel<DOWN, B>);
    const size_t smem = gemm_tc_smem_bytes();
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    GemmArgs copy = a;
    void* args[] = {&copy};
    return launch_pdl_raw(fn, dim3(sms), dim3(kThreads), smem, stream, args);
}

template <bool DOWN>
static cudaError_t launch_b(const GemmArgs& a, cudaStream_t stream, int sms) {
    switch (a.B) {
        case 1: return launch_one<DOWN, 1>(a, stream, sms);
        case 2: return launch_one<DOWN, 2>(a, stream, sms);
        case 3: return launch_one<DOWN, 3>(a, stream, sms);
        case 4: return launch_one<DOWN, 4>(a, stream, sms);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm_gateup(const GemmArgs& a, cudaStream_t stream, int sms) { return launch_b<false>(a, stream, sms); }
cudaError_t launch_gemm_down(const GemmArgs& a, cudaStream_t stream, int sms) { return launch_b<true>(a, stream, sms); }

}  // namespace dpa
