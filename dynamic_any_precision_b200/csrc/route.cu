// Router: softmax top-k gating (DPA-MoE abstract: each token is routed to a small set of
// experts; the gate scores then drive the plane allocation).
//
// The routing decision has to be reproducible bit for bit by any IEEE implementation, so:
//  * the logit is the exact dot product of the bf16 token and the bf16 router row, rounded
//    once to fp64. Products of two bf16 values are exact in fp64. A warp sums them in fp64 in
//    any order and proves the sum exact (every product is a multiple of 2^L, L = lowest set
//    bit of any operand pair, and sum|p| < 2^(L+52), so no partial sum can round). If the
//    proof fails (operands spread over more than ~50 binades), the warp redoes the dot
//    product in a 544-bit fixed-point accumulator and rounds that once.
//  * exp is one fixed fp64 procedure (Cody & Waite reduction with ln 2 in two parts, degree-13
//    Taylor polynomial in Horner form, scaling by 2^n), every step an explicitly rounded
//    fp64 operation (this file is also compiled with --fmad=false).
// The last block to finish a token (atomic ticket) selects its top-k and computes the gates,
// and block 0 of each token writes the token's fixed-point digits for the expert GEMV.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kRouteWarps = 8;
// Router-row uint4 loads a lane issues at once (PF, a template parameter of the per-logit kernel):
// the number a lane needs in total when that is at most 8, so that no unrolled slot idles.
constexpr int16_t kNoBit = 0x3FFF;   // lowest-set-bit marker of a zero element
#ifndef DPA_ROUTE_TILED_MIN_TOKENS
#define DPA_ROUTE_TILED_MIN_TOKENS 2
#endif
constexpr int kRouteTiledMinTokens = DPA_ROUTE_TILED_MIN_TOKENS;   // from here on the logits run as a tiled GEMM
constexpr int kMaxLsbBlocks = 256;          // H <= 16384 on the tiled path

// ---------------- fp64 exp (see header comment) ----------------
__device__ __forceinline__ double dexp_fixed(double x) {
    const double INV_LN2 = 0x1.71547652b82fep+0;
    const double LN2_HI = 0x1.62e42fefa3800p-1;
    const double LN2_LO = 0x1.ef35793c76730p-45;
    // 1/i!, i = 0..13, each rounded to nearest fp64
    const double C[14] = {0x1.0000000000000p+0, 0x1.0000000000000p+0, 0x1.0000000000000p-1,
                          0x1.5555555555555p-3, 0x1.5555555555555p-5, 0x1.1111111111111p-7,
                          0x1.6c16c16c16c17p-10, 0x1.a01a01a01a01ap-13, 0x1.a01a01a01a01ap-16,
                          0x1.71de3a556c734p-19, 0x1.27e4fb7789f5cp-22, 0x1.ae64567f544e4p-26,
                          0x1.1eed8eff8d898p-29, 0x1.6124613a86d09p-33};
    if (x < -708.0) return 0.0;
    const double nf = rint(__dmul_rn(x, INV_LN2));   // ties to even
    const int n = static_cast<int>(nf);
    const double r = __dsub_rn(__dsub_rn(x, __dmul_rn(nf, LN2_HI)), __dmul_rn(nf, LN2_LO));
    double p = C[13];
#pragma unroll
    for (int i = 12; i >= 0; --i) p = __dadd_rn(__dmul_rn(p, r), C[i]);
    // p * 2^n is exact here: n >= -1021 and p in [0.7, 1.42], so the result is normal.
    const double two_n = __longlong_as_double(static_cast<long long>(n + 1023) << 52);
    return __dmul_rn(p, two_n);
}

// ---------------- bf16 decomposition ----------------
struct Bf16Parts {
    int mant;   // integer significand (0..255), 0 for +-0
    int exp;    // value = mant * 2^exp
    int sign;
    bool finite;
};

__device__ __forceinline__ Bf16Parts bf16_parts(uint32_t u) {
    Bf16Parts p;
    const int E = (u >> 7) & 0xFF;
    const int M = u & 0x7F;
    p.sign = (u >> 15) & 1;
    p.finite = E != 0xFF;
    p.mant = E ? (M | 0x80) : M;
    p.exp = (E ? E : 1) - 134;
    return p;
}

// exponent of the lowest set bit of a nonzero bf16 value
__device__ __forceinline__ int bf16_lsb(uint32_t u) {
    const Bf16Parts p = bf16_parts(u);
    return p.exp + (__ffs(p.mant) - 1);
}

// exponent of the lowest set bit of a finite double (a large value for zero)
__device__ __forceinline__ int f64_lsb(double v) {
    const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(v));
    const int ef = static_cast<int>((b >> 52) & 0x7FF);
    unsigned long long m = b & 0xFFFFFFFFFFFFFull;
    if (ef) m |= 1ull << 52;
    return m ? (ef ? ef : 1) - 1075 + (__ffsll(static_cast<long long>(m)) - 1) : (1 << 20);
}

// 2^k as a double, k in [-1022, 1023]
__device__ __forceinline__ double pow2(int k) {
    return __longlong_as_double(static_cast<long long>(k + 1023) << 52);
}

// ---------------- exact fixed-point dot product (slow path) ----------------
// Products are m * 2^f with m < 2^16 and f in [-266, 240]; bit b = f + 266 in [0, 506].
constexpr int kLimbs = 17;   // 544 bits of 32-bit limbs held in int64 to absorb carries

__device__ double exact_dot_fixed(const uint16_t* xs, const uint16_t* w, int H, int lane) {
    long long limb[kLimbs];
#pragma unroll
    for (int i = 0; i < kLimbs; ++i) limb[i] = 0;
    for (int j = lane; j < H; j += 32) {
        const Bf16Parts a = bf16_parts(xs[j]);
        const Bf16Parts b = bf16_parts(w[j]);
        if (a.mant == 0 || b.mant == 0) continue;
        const int bit = a.exp + b.exp + 266;
        const long long v = static_cast<long long>(a.mant * b.mant) << (bit & 31);
        const int L = bit >> 5;
        if (a.sign ^ b.sign) limb[L] -= v; else limb[L] += v;
    }
#pragma unroll
    for (int i = 0; i < kLimbs; ++i) {
        long long v = limb[i];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        limb[i] = v;
    }
    // every lane now holds the same limbs; normalise to a two's-complement 544-bit integer
    uint32_t d[kLimbs];
    long long carry = 0;
    for (int i = 0; i < kLimbs; ++i) {
        const long long v = limb[i] + carry;
        d[i] = static_cast<uint32_t>(v & 0xffffffffll);
        carry = v >> 32;   // arithmetic shift: floor division
    }
    const bool neg = carry < 0;
    if (neg) {   // magnitude = -(value): invert and add one
        uint64_t c = 1;
        for (int i = 0; i < kLimbs; ++i) {
            const uint64_t s = static_cast<uint64_t>(~d[i]) + c;
            d[i] = static_cast<uint32_t>(s);
            c = s >> 32;
        }
    }
    int top = -1;
    for (int i = kLimbs - 1; i >= 0; --i)
        if (d[i]) { top = 32 * i + 31 - __clz(d[i]); break; }
    if (top < 0) return 0.0;
    auto bit_at = [&](int pos) -> uint32_t { return (d[pos >> 5] >> (pos & 31)) & 1u; };
    double mag;
    if (top <= 52) {
        uint64_t m = static_cast<uint64_t>(d[0]) | (static_cast<uint64_t>(d[1]) << 32);
        mag = __dmul_rn(static_cast<double>(m), pow2(-266));   // m < 2^53: exact
    } else {
        const int lo = top - 52;            // lowest kept bit
        uint64_t m = 0;
        for (int pos = top; pos >= lo; --pos) m = (m << 1) | bit_at(pos);
        const uint32_t rbit = bit_at(lo - 1);
        bool sticky = false;
        for (int pos = lo - 2; pos >= 0 && !sticky; --pos) sticky = bit_at(pos) != 0;
        int e = lo;
        if (rbit && (sticky || (m & 1))) {
            m += 1;
            if (m >> 53) { m >>= 1; e += 1; }
        }
        mag = __dmul_rn(static_cast<double>(m), pow2(e - 266));
    }
    return neg ? -mag : mag;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
    for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int warp_min_i(int v) {
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_max_f(float v) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int warp_sum_i(int v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Exact dot product of one (token, router row) pair by a warp: fp64 sum with the per-product
// lowest-bit proof (every product a multiple of 2^lmin, sum |p| < 2^(lmin+53)), else the
// fixed-point accumulator. Both operands are bf16 rows (global or shared memory, 16-byte
// aligned, H a multiple of 8); a lane takes 8 consecutive inputs per 16-byte load and issues
// up to 8 such loads per operand before using them.
__device__ double exact_dot_warp(const uint16_t* x, const uint16_t* w, int H, int lane) {
    double acc = 0.0, absacc = 0.0;
    int lmin = 1 << 20;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    const uint4* wv = reinterpret_cast<const uint4*>(w);
    const int nq = H >> 3;
    for (int q0 = 0; q0 < nq; q0 += 32 * 8) {
        uint4 xa[8], wa[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = q0 + 32 * u + lane;
            xa[u] = q < nq ? xv[q] : make_uint4(0, 0, 0, 0);
            wa[u] = q < nq ? wv[q] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t xw[4] = {xa[u].x, xa[u].y, xa[u].z, xa[u].w};
            const uint32_t ww[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                const uint32_t xu = (xw[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
                const uint32_t wu = (ww[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
                const double p = __dmul_rn(static_cast<double>(__uint_as_float(xu << 16)),
                                           static_cast<double>(__uint_as_float(wu << 16)));
                acc = __dadd_rn(acc, p);
                absacc = __dadd_rn(absacc, fabs(p));
                if ((xu & 0x7FFF) && (wu & 0x7FFF)) lmin = min(lmin, bf16_lsb(xu) + bf16_lsb(wu));
            }
        }
    }
    acc = warp_sum_f64(acc);
    absacc = warp_sum_f64(absacc);
    lmin = warp_min_i(lmin);
    if (absacc == 0.0) return acc;
    int ea;
    frexp(absacc, &ea);   // absacc < 2^ea
    if (ea <= lmin + 52) return acc;
    return exact_dot_fixed(x, w, H, lane);
}

// Fixed-point digits of token t for the expert GEMV: groups g = g0, g0 + gstep, ... handled by
// this warp; xs is the token's bf16 row (shared or global memory). Per group of G inputs,
// X = rint(x * 2^(14 - E)) with |x| < 2^E, stored as digits d0 + 256 d1 in rows [T][2][H] whose
// 64-column blocks are permuted (column c at byte 16*((c%16)/4) + 4*(c/16) + c%4) so that one
// 16-byte load gives an MMA lane its B-operand words; the group scales 2^(E-14) and scaled sums
// [T][ngp], ngp = H/G rounded up to a multiple of 4.
__device__ void token_digits(const RouteArgs& a, int t, const uint16_t* xs, int g0, int gstep) {
    const int H = a.H, G = a.G, ng = H / G, ngp = (ng + 3) & ~3, lane = threadIdx.x & 31;
    for (int g = g0; g < ng; g += gstep) {
        float mx = 0.f;
        for (int j = lane; j < G; j += 32) mx = fmaxf(mx, fabsf(bf16_bits_to_float(xs[g * G + j])));
        mx = warp_max_f(mx);
        const int Eg = group_exponent(mx);
        int sum = 0;
        for (int j = lane; j < G; j += 32) {
            const int c = g * G + j;
            const int X = __float2int_rn(ldexpf(bf16_bits_to_float(xs[c]), 14 - Eg));
            sum += X;
            const int lo = ((X + 128) & 255) - 128;
            const int hi = (X - lo) >> 8;
            const int cb = c & 63;
            const size_t off = static_cast<size_t>(t) * 2 * H + (c & ~63) + 16 * ((cb & 15) >> 2) + 4 * (cb >> 4) + (cb & 3);
            a.xdig[off] = static_cast<int8_t>(lo);
            a.xdig[off + H] = static_cast<int8_t>(hi);
        }
        sum = warp_sum_i(sum);
        if (lane == 0) {   // |sum| <= G 2^14 <= 2^23: the scaled sum is exact in fp32
            const float scl = ldexpf(1.f, Eg - 14);
            a.xscl[t * ngp + g] = scl;
            a.xfsx[t * ngp + g] = scl * static_cast<float>(sum);
        }
    }
}

// ---- top-k by warp extraction (E <= 32 w experts on the first w warps, w K <= 32) ----
// A logit as an order-preserving 64-bit key: larger logit, larger key; -0 ties with +0; NaN is
// below every number.
__device__ __forceinline__ unsigned long long logit_key(double v) {
    if (v != v) return 0ull;
    const unsigned long long b = v == 0.0 ? 0ull : static_cast<unsigned long long>(__double_as_longlong(v));
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
// The K largest keys among the lanes with `avail`, largest first, equal keys by lowest lane:
// lane r < K receives the r-th key and the lane that held it (ok false: none was left).
__device__ __forceinline__ void warp_extract(unsigned long long key, bool avail, int K, int lane,
                                             unsigned long long& out_key, int& out_lane, bool& out_ok) {
    out_key = 0ull;
    out_lane = 0;
    out_ok = false;
    for (int r = 0; r < K; ++r) {
        const uint32_t hi = avail ? static_cast<uint32_t>(key >> 32) : 0u;
        const uint32_t mh = __reduce_max_sync(0xffffffffu, hi);
        const bool c1 = avail && hi == mh;
        const uint32_t lo = c1 ? static_cast<uint32_t>(key) : 0u;
        const uint32_t ml = __reduce_max_sync(0xffffffffu, lo);
        const unsigned c2 = __ballot_sync(0xffffffffu, c1 && static_cast<uint32_t>(key) == ml);
        const int win = __ffs(static_cast<int>(c2)) - 1;
        if (lane == r) {
            out_ok = win >= 0;
            out_lane = win >= 0 ? win : 0;
            out_key = (static_cast<unsigned long long>(mh) << 32) | ml;
        }
        if (lane == win) avail = false;
    }
}
// Each of the first w warps extracts the K largest of its 32 experts; warp 0 extracts the K
// largest of those w K candidates (laid out by warp, then in extraction order, so equal keys
// stay in ascending expert id), then computes the gates with shuffles. The same order and the
// same arithmetic as the rank-based path below. Returns false (before any work) where the
// shape does not fit; the decision is uniform over the block.
__device__ bool select_topk_gates_warp(const RouteArgs& a, int t, const double* lrow, unsigned char* smem_raw) {
    __shared__ unsigned long long s_ck[32];
    __shared__ double s_cv[32];
    __shared__ int s_ce[32], s_cok[32];
    __shared__ double s_lmax, s_den;
    const int E = a.E, K = a.K;
    const int nwu = (E + 31) >> 5;
    if (K > 32 || nwu * K > 32 || nwu * 32 > static_cast<int>(blockDim.x)) return false;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double v = 0.0;
    if (warp < nwu) {
        const int e = warp * 32 + lane;
        const bool valid = e < E;
        v = valid ? __ldcg(lrow + e) : 0.0;
        unsigned long long ck;
        int cl;
        bool ok;
        warp_extract(valid ? logit_key(v) : 0ull, valid, K, lane, ck, cl, ok);
        const double cv = __shfl_sync(0xffffffffu, v, cl);
        if (lane < K) {
            s_ck[warp * K + lane] = ck;
            s_cv[warp * K + lane] = cv;
            s_ce[warp * K + lane] = warp * 32 + cl;
            s_cok[warp * K + lane] = ok ? 1 : 0;
        }
    }
    __syncthreads();
    double num = 0.0, vs = 0.0;
    int es = 0;
    if (warp == 0) {
        const bool have = lane < nwu * K && s_cok[lane] != 0;
        unsigned long long fk;
        int fl;
        bool ok;
        warp_extract(have ? s_ck[lane] : 0ull, have, K, lane, fk, fl, ok);
        es = s_ce[fl];
        vs = s_cv[fl];
        const double lmax = __shfl_sync(0xffffffffu, vs, 0);
        if (lane < K) num = dexp_fixed(__dsub_rn(vs, lmax));
        if (lane == 0) s_lmax = lmax;
    }
    if (!a.norm_topk) {   // the denominator sums every expert's exp, in expert order
        double* ex = reinterpret_cast<double*>(smem_raw);   // [E]
        __syncthreads();
        if (warp < nwu && warp * 32 + lane < E) ex[warp * 32 + lane] = dexp_fixed(__dsub_rn(v, s_lmax));
        __syncthreads();
        if (threadIdx.x == 0) {
            double den = 0.0;
            for (int i = 0; i < E; ++i) den = __dadd_rn(den, ex[i]);
            s_den = den;
        }
        __syncthreads();
    }
    if (warp == 0) {
        double den = 0.0;
        if (a.norm_topk) {
            for (int j = 0; j < K; ++j) den = __dadd_rn(den, __shfl_sync(0xffffffffu, num, j));
        } else {
            den = s_den;
        }
        if (lane < K) {
            a.idx[t * K + lane] = es;
            a.gate[t * K + lane] = __ddiv_rn(num, den);
        }
    }
    return true;
}

// Top-k by exact fp64 logit (descending, ties to the lower expert id, NaN last) and the gates
// (fixed fp64 exp; softmax over the top-k or over all experts). Whole block; smem_raw holds at
// least 24 * E bytes.
__device__ void select_topk_gates(const RouteArgs& a, int t, unsigned char* smem_raw) {
    __shared__ int s_sel[32];
    __shared__ double s_num[32];
    __shared__ double s_den;
    const int E = a.E;
    // the logits were written by other blocks or kernels (fenced / completed); read them from L2
    const double* lrow = (a.logits_user ? a.logits_user : a.logits_ws) + static_cast<size_t>(t) * E;
    if (select_topk_gates_warp(a, t, lrow, smem_raw)) return;
    double* vals = reinterpret_cast<double*>(smem_raw);             // [E] logits (token no longer needed)
    float* fk = reinterpret_cast<float*>(vals + E);                 // [E] fp32 roundings of the logits
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        const double v = __ldcg(lrow + i);
        vals[i] = v;
        fk[i] = v == v ? __double2float_rn(v) : -INFINITY;   // NaN is never larger
    }
    __syncthreads();
    const int K = a.K;
    // rank of each expert = number of experts before it (descending logit, ties to the lower
    // id; NaN ranks last, NaNs by id). Q threads share a candidate, each counting over 1/Q of
    // the experts. The ranks are a permutation of 0..E-1, so s_sel[0..K) is always written.
    int Q = 1;
    while (Q < 32 && Q * 2 * E <= static_cast<int>(blockDim.x)) Q *= 2;
    const int chunk = (E + Q - 1) / Q;
    for (int base = 0; base < E * Q; base += blockDim.x) {
        const int idx = base + threadIdx.x;
        const int c = idx / Q, q = idx % Q;
        int rank = 0;
        if (c < E) {
            const double v = vals[c];
            if (v == v) {
                // fp32 rounding is monotone: fk[j] > fk[c] implies vals[j] > vals[c]; only equal fp32
                // values need the exact fp64 comparison (with ties to the lower expert id)
                const float fv = fk[c];
                const int j0 = q * chunk, j1 = min(E, (q + 1) * chunk);
                int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
                int j = j0;
                for (; j + 4 <= j1; j += 4) {   // four independent comparisons per iteration
                    const float u0 = fk[j], u1 = fk[j + 1], u2 = fk[j + 2], u3 = fk[j + 3];
                    r0 += u0 > fv ? 1 : 0;
                    r1 += u1 > fv ? 1 : 0;
                    r2 += u2 > fv ? 1 : 0;
                    r3 += u3 > fv ? 1 : 0;
                    if (u0 == fv || u1 == fv || u2 == fv || u3 == fv) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int jj = j + u;
                            if (fk[jj] == fv && jj != c) {
                                const double w = vals[jj];
                                r0 += (w > v || (w == v && jj < c)) ? 1 : 0;
                            }
                        }
                    }
                }
                for (; j < j1; ++j) {
                    const float u = fk[j];
                    r0 += u > fv ? 1 : 0;
                    if (u == fv && j != c) {
                        const double w = vals[j];
                        r0 += (w > v || (w == v && j < c)) ? 1 : 0;
                    }
                }
                rank = (r0 + r1) + (r2 + r3);
            } else {
                // a NaN logit (a non-finite token or router weight, flagged as invalid input)
                // ranks after every number and after the NaNs of lower id, so that the ranks
                // stay a permutation and every selected slot holds a valid expert id
                const int j0 = q * chunk, j1 = min(E, (q + 1) * chunk);
                int r = 0;
                for (int j = j0; j < j1; ++j) {
                    const double w = vals[j];
                    r += (w == w || j < c) ? 1 : 0;
                }
                rank = r;
            }
        }
        for (int o = 1; o < Q; o <<= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
        if (c < E && q == 0 && rank < K) s_sel[rank] = c;
    }
    __syncthreads();
    const double lmax = vals[s_sel[0]];
    if (threadIdx.x < K) s_num[threadIdx.x] = dexp_fixed(__dsub_rn(vals[s_sel[threadIdx.x]], lmax));
    double* ex = vals + 2 * E;   // [E] exp values (norm over all experts), after the fp32 keys
    if (!a.norm_topk)
        for (int i = threadIdx.x; i < E; i += blockDim.x) ex[i] = dexp_fixed(__dsub_rn(vals[i], lmax));
    __syncthreads();
    if (threadIdx.x == 0) {
        double den = 0.0;
        if (a.norm_topk) {
            for (int j = 0; j < K; ++j) den = __dadd_rn(den, s_num[j]);
        } else {
            for (int i = 0; i < E; ++i) den = __dadd_rn(den, ex[i]);
        }
        s_den = den;
    }
    __syncthreads();
    if (threadIdx.x < K) {
        a.idx[t * K + threadIdx.x] = s_sel[threadIdx.x];
        a.gate[t * K + threadIdx.x] = __ddiv_rn(s_num[threadIdx.x], s_den);
    }
}

template <int PF>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(RouteArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int H = a.H, E = a.E, H8 = H >> 3;
    // token in lane-major order: element j lives at (j & 7) * H8 + (j >> 3), so the 8
    // consecutive elements a lane multiplies sit in 8 conflict-free rows
    double* xd = reinterpret_cast<double*>(smem_raw);                 // [H]
    int16_t* xl = reinterpret_cast<int16_t*>(xd + H);                 // [H] lowest set bit (kNoBit: zero)
    uint16_t* xs = reinterpret_cast<uint16_t*>(xl + H);               // [H] bf16 bits (natural order)
    __shared__ int s_last;
    __shared__ double s_acc[kRouteWarps], s_abs[kRouteWarps];
    __shared__ int s_lmin[kRouteWarps], s_bad[kRouteWarps];
    const int t = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wpe = a.wpe;                    // warps per expert (1, 2, 4 or 8)
    const int part = warp % wpe;
    const uint16_t* xrow = a.x + static_cast<size_t>(t) * H;

    // this warp's router-row loads go out first, so they overlap the staging of the token
    const int e = blockIdx.x * (kRouteWarps / wpe) + warp / wpe;
    const int wstride = 32 * wpe;                       // uint4 columns per round
    const int nq = (H8 + wstride - 1) / wstride;
    uint4 wpre[PF];
    if (e < E) {
        const uint4* wrow = reinterpret_cast<const uint4*>(a.wr + static_cast<size_t>(e) * H);
#pragma unroll
        for (int u = 0; u < PF; ++u) {
            const int col = u * wstride + part * 32 + lane;
            if (u < nq && col < H8) wpre[u] = wrow[col];
        }
    }

    // the token and the workspace may come from the previous kernel: wait for it from here on
    pdl_wait();

    // stage the token: each thread loads up to 4 x 8 elements with all loads issued first
    bool bad = false;
    for (int c0 = threadIdx.x; c0 < H8; c0 += 4 * blockDim.x) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = c0 + u * blockDim.x;
            if (c < H8) v[u] = reinterpret_cast<const uint4*>(xrow)[c];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = c0 + u * blockDim.x;   // 8-element group index
            if (c < H8) {
                const uint32_t ww[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    const uint16_t xu = static_cast<uint16_t>((ww[h >> 1] >> (16 * (h & 1))) & 0xFFFFu);
                    const int q = h * H8 + c;
                    xd[q] = static_cast<double>(bf16_bits_to_float(xu));
                    xl[q] = (xu & 0x7FFF) ? static_cast<int16_t>(bf16_lsb(xu)) : kNoBit;
                    bad |= ((xu >> 7) & 0xFF) == 0xFF;
                }
                reinterpret_cast<uint4*>(xs)[c] = v[u];
            }
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 1);

    // ---- wpe warps per expert logit: partial sums of products, lowest bits, magnitudes ----
    {
        double acc0 = 0.0, acc1 = 0.0, abs0 = 0.0, abs1 = 0.0;
        int lmin = 1 << 20;
        bool wbad = false;
        if (e < E) {
            const uint4* wrow = reinterpret_cast<const uint4*>(a.wr + static_cast<size_t>(e) * H);
            for (int q0 = 0; q0 < nq; q0 += PF) {
                uint4 wv[PF];
#pragma unroll
                for (int u = 0; u < PF; ++u) {
                    const int col = (q0 + u) * wstride + part * 32 + lane;
                    if (q0 == 0) wv[u] = wpre[u];
                    else if (q0 + u < nq && col < H8) wv[u] = wrow[col];
                }
#pragma unroll
                for (int u = 0; u < PF; ++u) {
                    const int col = (q0 + u) * wstride + part * 32 + lane;   // 8-element group index
                    if (q0 + u < nq && col < H8) {
                        const uint32_t ww[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            const uint32_t wu = (ww[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
                            const double xv = xd[h * H8 + col];
                            const double p = __dmul_rn(xv, static_cast<double>(__uint_as_float(wu << 16)));
                            if (h & 1) { acc1 = __dadd_rn(acc1, p); abs1 = __dadd_rn(abs1, fabs(p)); }
                            else { acc0 = __dadd_rn(acc0, p); abs0 = __dadd_rn(abs0, fabs(p)); }
                            if (wu & 0x7FFF) lmin = min(lmin, static_cast<int>(xl[h * H8 + col]) + bf16_lsb(wu));
                            wbad |= ((wu >> 7) & 0xFF) == 0xFF;
                        }
                    }
                }
            }
        }
        const double acc = warp_sum_f64(__dadd_rn(acc0, acc1));
        const double absacc = warp_sum_f64(__dadd_rn(abs0, abs1));
        lmin = warp_min_i(lmin);
        wbad = __any_sync(0xffffffffu, wbad);
        if (lane == 0) {
            s_acc[warp] = acc;
            s_abs[warp] = absacc;
            s_lmin[warp] = lmin;
            s_bad[warp] = wbad ? 1 : 0;
        }
    }
    __syncthreads();
    if (part == 0 && e < E) {
        // combine the expert's partial sums (exact whenever the bound below holds)
        double acc = s_acc[warp], absacc = s_abs[warp];
        int lmin = s_lmin[warp], wbad = s_bad[warp];
        for (int w = 1; w < wpe; ++w) {
            acc = __dadd_rn(acc, s_acc[warp + w]);
            absacc = __dadd_rn(absacc, s_abs[warp + w]);
            lmin = min(lmin, s_lmin[warp + w]);
            wbad |= s_bad[warp + w];
        }
        double logit = acc;
        if (absacc != 0.0) {
            int ea;
            frexp(absacc, &ea);   // absacc < 2^ea
            // every product is a multiple of 2^lmin and sum |p| < 2^(lmin+53): no partial sum
            // in any order can round, so acc is the exact dot product. Otherwise recompute.
            if (ea > lmin + 52) logit = exact_dot_fixed(xs, a.wr + static_cast<size_t>(e) * H, H, lane);
        }
        if (lane == 0) {
            double* dst = a.logits_user ? a.logits_user : a.logits_ws;
            dst[static_cast<size_t>(t) * E + e] = logit;
            if (wbad) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 2);
        }
    }

    // ---- fixed-point digits of x for the expert GEMV: the token's blocks share the groups ----
    if (a.xdig != nullptr) token_digits(a, t, xs, blockIdx.x + warp * gridDim.x, gridDim.x * kRouteWarps);

    // ---- last block of this token: top-k and gates ----
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&a.counters[t], 1u);
        s_last = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    if (threadIdx.x == 0) a.counters[t] = 0;   // ready for the next call

    select_topk_gates(a, t, smem_raw);
}


// ---------------- large batches: logits as a tiled fp64 GEMM ----------------
// Exactness without per-product bookkeeping. Split the H inputs into blocks b of 64. Every
// product x_j * w_j of block b is a multiple of 2^(Lx_b + Lw_b) (lowest set bit over the block's
// nonzero elements of the token / the router row). Two tests, either of which proves that the
// logit the selection kernel sums is the exact dot product:
//  - whole row: every product is a multiple of 2^L with L = min_b (Lx_b + Lw_b), and by
//    Cauchy-Schwarz every partial sum, in any order, is at most |x| |w|. If
//    |x|^2 |w|^2 < 2^(2 (L + 53)), every partial sum is a multiple of 2^L below 2^(L+53): exact.
//  - per slice, then across slices: a slice of the tiled GEMM touches blocks b0..b1; its
//    products are multiples of 2^Ls, Ls = min (Lx_b + Lw_b) over those blocks, and each of its
//    partial sums is at most sum_b |x_b| |w_b| < (b1 - b0 + 1) 2^Hs with |x_b| < 2^hx_b,
//    |w_b| < 2^hw_b, Hs = max (hx_b + hw_b). If that bound is at most 2^(Ls+53), the slice sum
//    is exact. The exact slice sums v_s are then multiples of 2^m (m: the lowest set bit over
//    the nonzero v_s, read from their bits) and their partial sums are at most sum_s |v_s|; if
//    that is below 2^(m+53), the sum over the slices is exact too. This test only fails where
//    one slice really spans more than 53 bits, where the whole-row test fails for any token
//    with one tiny element.
// Logits for which both tests fail are recomputed by the selection kernel with the per-product
// proof and, failing that, the fixed-point dot product, so the result is always the exact dot
// product rounded once, as in the per-logit kernel.

constexpr int kNoLsb = 0x3FFF;      // block (or row) without a nonzero element
constexpr int kLsbBlock = 64;       // inputs per lowest-bit block

// One CTA per row (tokens 0..T-1, then router rows): per-block lowest set bit and norm
// exponent, sum of squares, NaN/Inf flag. Any block of up to 8 warps.
__device__ void route_stats_row(const RouteArgs& a, int r) {
    __shared__ double s_n[8];
    __shared__ int s_b[8];
    const int H = a.H, nb = H / kLsbBlock;
    const bool is_tok = r < a.T;
    const size_t ro = static_cast<size_t>(is_tok ? r : r - a.T) * nb;
    const uint16_t* row = is_tok ? a.x + static_cast<size_t>(r) * H : a.wr + static_cast<size_t>(r - a.T) * H;
    int16_t* lrow = (is_tok ? a.lsb_x : a.lsb_w) + ro;
    int16_t* hrow = (is_tok ? a.hb_x : a.hb_w) + ro;
    int bad = 0;
    double n2 = 0.0;
    // thread c covers elements 8c .. 8c+7; 8 consecutive lanes make one block of 64
    for (int c0 = 0; c0 < H / 8; c0 += blockDim.x) {
        const int c = c0 + threadIdx.x;
        int l = kNoLsb;
        double q = 0.0;   // this thread's part of the block's sum of squares
        if (c < H / 8) {
            const uint4 v = reinterpret_cast<const uint4*>(row)[c];
            const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                const uint32_t u = (ww[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
                if (u & 0x7FFF) l = min(l, bf16_lsb(u));
                bad |= ((u >> 7) & 0xFF) == 0xFF;
                const double d = static_cast<double>(__uint_as_float(u << 16));
                q = __dadd_rn(q, __dmul_rn(d, d));
            }
        }
        n2 = __dadd_rn(n2, q);
        for (int o = 1; o < 8; o <<= 1) {
            l = min(l, __shfl_xor_sync(0xffffffffu, l, o));
            q = __dadd_rn(q, __shfl_xor_sync(0xffffffffu, q, o));
        }
        if (c < H / 8 && (c & 7) == 0) {
            // squares of bf16 values are exact; 63 roundings of the sum stay below 2^-46
            // relative, so q (1 + 2^-40) bounds the block's sum of squares from above; with
            // q (1 + 2^-40) < 2^ex, the block's norm is below 2^ceil(ex / 2)
            int hb = -kNoLsb;
            if (q > 0.0) {
                int ex;
                frexp(__dmul_rn(q, 1.0 + 0x1p-40), &ex);
                hb = (ex + 1) >> 1;
            }
            lrow[c >> 3] = static_cast<int16_t>(l);
            hrow[c >> 3] = static_cast<int16_t>(hb);
        }
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    n2 = warp_sum_f64(n2);
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) { s_n[warp] = n2; s_b[warp] = bad; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < nw; ++w) { n2 = __dadd_rn(n2, s_n[w]); bad |= s_b[w]; }
        if (is_tok) a.n2_x[r] = n2;
        else a.n2_w[r - a.T] = n2;
        if (bad) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, is_tok ? 1 : 2);
    }
}

constexpr int kGK = 32;            // inputs per k stage of the tiled logits
constexpr int kGThreads = 256;     // 8 warps: 4 token quarters x 2 expert halves of the CTA tile

__device__ __forceinline__ double bf16_to_f64(uint32_t u) { return static_cast<double>(__uint_as_float(u << 16)); }

// Tiled logits: CTA tile TT tokens x TE experts over one slice of the inputs, fp64 FMAs (every
// product of two bf16 values is exact in fp64; the sums are exact whenever the bound above
// holds, which the selection kernel checks). Each thread owns TT/16 tokens x TE/16 experts.
// Grid (ceil(T/TT), ceil(E/TE), ks); the slice sums go to part[ks][T][E] (no atomics; the
// selection kernel adds the ks slices of a logit).
template <int TT, int TE>
__device__ __forceinline__ void route_gemm_tile(const RouteArgs& a, int kslice, int bx, int by, int bz,
                                                unsigned char* smem_raw) {
    constexpr int MT = TT / 16, ME = TE / 16;
    double* sx = reinterpret_cast<double*>(smem_raw);          // [2][kGK][TT]
    double* sw = sx + 2 * kGK * TT;                             // [2][kGK][TE]
    const int H = a.H, T = a.T, E = a.E;
    const int t0 = bx * TT, e0 = by * TE;
    const int k0 = bz * kslice, k1 = min(H, k0 + kslice);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wt = warp & 3, we = warp >> 2, tg = lane & 3, eg = lane >> 2;
    const int tb = (TT / 4) * wt + MT * tg, eb = (TE / 2) * we + ME * eg;   // this thread's tokens, experts

    // staging: the x tile (TT rows x 32 inputs) and the w tile (TE rows x 32), 8 inputs per uint4
    constexpr int NXL = (TT * 4 + kGThreads - 1) / kGThreads, NWL = (TE * 4 + kGThreads - 1) / kGThreads;
    uint4 rx[NXL], rw[NWL];
    auto load = [&](int kc) {
#pragma unroll
        for (int u = 0; u < NXL; ++u) {
            const int i = tid + u * kGThreads, xt = i % TT, xk = (i / TT) * 8;
            rx[u] = make_uint4(0, 0, 0, 0);
            if (i < TT * 4 && t0 + xt < T) rx[u] = *reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0 + xt) * H + kc + xk);
        }
#pragma unroll
        for (int u = 0; u < NWL; ++u) {
            const int i = tid + u * kGThreads, wi = i % TE, wk = (i / TE) * 8;
            rw[u] = make_uint4(0, 0, 0, 0);
            if (i < TE * 4 && e0 + wi < E) rw[u] = *reinterpret_cast<const uint4*>(a.wr + static_cast<size_t>(e0 + wi) * H + kc + wk);
        }
    };
    auto store = [&](int buf) {
        double* bx = sx + buf * kGK * TT;
        double* bw = sw + buf * kGK * TE;
#pragma unroll
        for (int u = 0; u < NXL; ++u) {
            const int i = tid + u * kGThreads, xt = i % TT, xk = (i / TT) * 8;
            if (i < TT * 4) {
                const uint32_t v[4] = {rx[u].x, rx[u].y, rx[u].z, rx[u].w};
#pragma unroll
                for (int h = 0; h < 8; ++h) bx[(xk + h) * TT + xt] = bf16_to_f64((v[h >> 1] >> (16 * (h & 1))) & 0xFFFFu);
            }
        }
#pragma unroll
        for (int u = 0; u < NWL; ++u) {
            const int i = tid + u * kGThreads, wi = i % TE, wk = (i / TE) * 8;
            if (i < TE * 4) {
                const uint32_t v[4] = {rw[u].x, rw[u].y, rw[u].z, rw[u].w};
#pragma unroll
                for (int h = 0; h < 8; ++h) bw[(wk + h) * TE + wi] = bf16_to_f64((v[h >> 1] >> (16 * (h & 1))) & 0xFFFFu);
            }
        }
    };

    double acc[MT][ME];
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < ME; ++j) acc[i][j] = 0.0;

    int buf = 0;
    load(k0);
    store(0);
    __syncthreads();
    for (int kc = k0; kc < k1; kc += kGK) {
        const bool more = kc + kGK < k1;
        if (more) load(kc + kGK);
        const double* bx = sx + buf * kGK * TT;
        const double* bw = sw + buf * kGK * TE;
#pragma unroll 4
        for (int k = 0; k < kGK; ++k) {
            double xv[MT], wv[ME];
#pragma unroll
            for (int i = 0; i < MT; i += 2) {
                if (i + 1 < MT) {
                    const double2 v = *reinterpret_cast<const double2*>(bx + k * TT + tb + i);
                    xv[i] = v.x;
                    xv[i + 1] = v.y;
                } else {
                    xv[i] = bx[k * TT + tb + i];
                }
            }
#pragma unroll
            for (int j = 0; j < ME; j += 2) {
                const double2 v = *reinterpret_cast<const double2*>(bw + k * TE + eb + j);
                wv[j] = v.x;
                wv[j + 1] = v.y;
            }
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int j = 0; j < ME; ++j) acc[i][j] = __fma_rn(xv[i], wv[j], acc[i][j]);
        }
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    double* dst = a.part + static_cast<size_t>(bz) * T * E;
#pragma unroll
    for (int i = 0; i < MT; ++i) {
        const int t = t0 + tb + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < ME; ++j) {
            const int e = e0 + eb + j;
            if (e < E) dst[static_cast<size_t>(t) * E + e] = acc[i][j];
        }
    }
}

// The router's first launch: three independent jobs side by side, by block index: the tiled
// logits (gx * gy * ks tiles), the exactness statistics of every token and router row (T + E
// rows), and the tokens' fixed-point digits for the expert GEMV (T tokens, when requested).
template <int TT, int TE>
__global__ void __launch_bounds__(kGThreads) route_prep_kernel(RouteArgs a, int kslice, int gx, int gy, int ks) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    pdl_wait();
    const int n_gemm = gx * gy * ks;
    const int b = blockIdx.x;
    if (b < n_gemm) {
        route_gemm_tile<TT, TE>(a, kslice, b % gx, (b / gx) % gy, b / (gx * gy), smem_raw);
    } else if (b < n_gemm + a.T + a.E) {
        route_stats_row(a, b - n_gemm);
    } else {
        const int t = b - n_gemm - a.T - a.E;
        token_digits(a, t, a.x + static_cast<size_t>(t) * a.H, threadIdx.x >> 5, kGThreads / 32);
    }
}

// One CTA per token (16 warps for small batches, so that a token's recomputed logits run at
// once; 4 for large ones, so that several tokens share an SM): check each logit's exactness
// bound, recompute the failures with
// the exact dot product, then top-k and gates.
constexpr int kSelWarpsMax = 16;
constexpr int kSelSmallBatch = 256;   // up to this many tokens: kSelWarpsMax warps per token
__global__ void __launch_bounds__(kSelWarpsMax * 32) route_select_kernel(RouteArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int s_fail[256];
    __shared__ int s_nfail;
    __shared__ int16_t s_lx[kMaxLsbBlocks], s_hx[kMaxLsbBlocks];
    pdl_wait();
    const int t = blockIdx.x, E = a.E, H = a.H, nb = H / kLsbBlock;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double* dst = (a.logits_user ? a.logits_user : a.logits_ws) + static_cast<size_t>(t) * E;
    if (threadIdx.x == 0) s_nfail = 0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
        s_lx[b] = a.lsb_x[static_cast<size_t>(t) * nb + b];
        s_hx[b] = a.hb_x[static_cast<size_t>(t) * nb + b];
    }
    __syncthreads();
    const double nx = a.n2_x[t];
    const int kslice = H / a.ks;   // inputs per slice of the tiled logits
    // tpe threads per expert (a power of two up to 4, neighbours in one warp): each takes the
    // slices sl = sub, sub + tpe, ... with the blocks they cover. Both exactness tests hold for
    // any order of the additions, so the partial sums may be combined in any order; a logit that
    // passes neither test is recomputed below.
    int tpe = 1;
    while (tpe < 4 && tpe * 2 * E <= static_cast<int>(blockDim.x)) tpe *= 2;
    const int sub = threadIdx.x & (tpe - 1);
    const size_t qs = static_cast<size_t>(a.T) * E;
    for (int g0 = 0; g0 < E * tpe; g0 += blockDim.x) {   // warp-uniform trip count
        const int e = (g0 + static_cast<int>(threadIdx.x)) / tpe;
        const bool act = e < E;
        const int16_t* lw = a.lsb_w + static_cast<size_t>(act ? e : 0) * nb;
        const int16_t* hw = a.hb_w + static_cast<size_t>(act ? e : 0) * nb;
        double v = 0.0, av = 0.0;   // this thread's slices: sum, sum of magnitudes
        int mv = 1 << 20;           //   lowest set bit over the nonzero slice sums
        int L = 2 * kNoLsb;         //   lowest product bit over their blocks (whole-row test)
        if (act) {
            const double* pe = a.part + static_cast<size_t>(t) * E + e;
            for (int q0 = sub; q0 < a.ks; q0 += 32 * tpe) {
                double u[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) u[j] = q0 + j * tpe < a.ks ? __ldcg(pe + (q0 + j * tpe) * qs) : 0.0;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    v = __dadd_rn(v, u[j]);
                    av = __dadd_rn(av, fabs(u[j]));
                    mv = min(mv, f64_lsb(u[j]));
                }
            }
            if (tpe == 1) {   // every block, eight at a time (nb is a multiple of 8: H % 512 == 0)
#pragma unroll 4
                for (int b0 = 0; b0 < nb; b0 += 8) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(lw + b0);
                    const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const int lv = static_cast<int16_t>((ww[h >> 1] >> (16 * (h & 1))) & 0xFFFFu);
                        L = min(L, static_cast<int>(s_lx[b0 + h]) + lv);
                    }
                }
            } else {          // the blocks of this thread's slices
                for (int sl = sub; sl < a.ks; sl += tpe) {
                    const int b0 = (sl * kslice) / kLsbBlock, b1 = ((sl + 1) * kslice - 1) / kLsbBlock;
                    for (int b = b0; b <= b1; ++b) L = min(L, static_cast<int>(s_lx[b]) + static_cast<int>(lw[b]));
                }
            }
        }
        for (int o = 1; o < tpe; o <<= 1) {   // the expert's threads meet (every lane takes part)
            v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            av = __dadd_rn(av, __shfl_xor_sync(0xffffffffu, av, o));
            mv = min(mv, __shfl_xor_sync(0xffffffffu, mv, o));
            L = min(L, __shfl_xor_sync(0xffffffffu, L, o));
        }
        // whole-row test (the same verdict in every thread of the expert): every product a
        // multiple of 2^L, every partial sum below |x| |w|
        bool ok = true;
        if (act && L < kNoLsb) {   // some block has nonzero products (else the logit is exactly 0)
            const int L2 = 2 * (L + 53);
            // margin 2^-20 covers the rounding of the two fp64 sums of squares
            const double lhs = __dmul_rn(__dmul_rn(nx, a.n2_w[e]), 1.0 + 0x1p-20);
            ok = L2 >= 1024 || (L2 > -1022 && lhs < pow2(L2));
        }
        // else each slice exact on its own (this thread's slices), then the sum over the slices
        bool oks = true;
        if (act && !ok) {
            for (int sl = sub; sl < a.ks && oks; sl += tpe) {
                const int b0 = (sl * kslice) / kLsbBlock, b1 = ((sl + 1) * kslice - 1) / kLsbBlock;
                int Ls = kNoLsb, Hs = -kNoLsb;
                for (int b = b0; b <= b1; ++b) {
                    const int lx = s_lx[b], lwb = lw[b];
                    if (lx < kNoLsb && lwb < kNoLsb) {   // both blocks hold nonzero elements
                        Ls = min(Ls, lx + lwb);
                        Hs = max(Hs, static_cast<int>(s_hx[b]) + static_cast<int>(hw[b]));
                    }
                }
                const int nbt = b1 - b0 + 1;
                const int cl = nbt > 1 ? 32 - __clz(nbt - 1) : 0;   // ceil(log2 nbt)
                oks = Ls >= kNoLsb || Hs + cl <= Ls + 53;
            }
        }
        for (int o = 1; o < tpe; o <<= 1) oks = (__shfl_xor_sync(0xffffffffu, oks ? 1 : 0, o) != 0) && oks;
        if (act && sub == 0) {
            dst[e] = v;
            if (!ok && oks) {
                if (av > 0.0) {
                    // the partial sums of the slice sums are multiples of 2^mv and at most av
                    // (summed with at most 255 roundings; 2^-40 bounds them)
                    int ea;
                    frexp(__dmul_rn(av, 1.0 + 0x1p-40), &ea);
                    ok = ea <= mv + 53;
                } else {
                    ok = true;   // every slice sum is zero: the logit is exactly 0
                }
            }
            if (!ok) {
                const int slot = atomicAdd(&s_nfail, 1);
                if (slot < 256) s_fail[slot] = e;
            }
        }
    }
    __syncthreads();
    const int nfail = s_nfail;
    const uint16_t* xrow = a.x + static_cast<size_t>(t) * H;
    if (nfail > 0) {
        // more failures than the list holds: recompute every logit of the token
        const int n = nfail <= 256 ? nfail : E;
        for (int i = warp; i < n; i += static_cast<int>(blockDim.x >> 5)) {
            const int e = nfail <= 256 ? s_fail[i] : i;
            const double v = exact_dot_warp(xrow, a.wr + static_cast<size_t>(e) * H, H, lane);
            if (lane == 0) dst[e] = v;
        }
        __syncthreads();
    }
    select_topk_gates(a, t, smem_raw);
}

}  // namespace

RouteTiling route_tiling(int T, int E, int H, int sms) {
    RouteTiling r;
    r.TT = T <= 16 ? 16 : 64;
    r.TE = T <= 64 ? 32 : 128;
    r.gx = (T + r.TT - 1) / r.TT;
    r.gy = (E + r.TE - 1) / r.TE;
    const int nchunks = H / kGK;
    int ks = 1;   // input slices: enough CTAs for every SM, each slice a whole number of k stages
    while (r.gx * r.gy * ks * 2 <= sms && ks * 2 <= nchunks && nchunks % (ks * 2) == 0) ks *= 2;
    r.ks = ks;
    r.kslice = (nchunks / ks) * kGK;
    return r;
}

bool route_tiled_path(int T, int H) {
    return T >= kRouteTiledMinTokens && H % kGK == 0 && H % (8 * kLsbBlock) == 0 && H / kLsbBlock <= kMaxLsbBlocks;
}

size_t route_partial_doubles(int T, int E, int H) {
    if (!route_tiled_path(T, H)) return 0;
    const RouteTiling r = route_tiling(T, E, H, kRouteMaxSms);
    return static_cast<size_t>(r.ks) * T * E;
}

template <int TT, int TE>
static cudaError_t launch_route_prep(RouteArgs& b, const RouteTiling& r, cudaStream_t stream) {
    const size_t smem = sizeof(double) * 2 * kGK * (TT + TE);
    const void* fn = reinterpret_cast<const void*>(route_prep_kernel<TT, TE>);
    // always raised: with the statistics role's static shared memory, 48 KB of dynamic does not fit
    // under the default limit
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    int kslice = r.kslice, gx = r.gx, gy = r.gy, ks = r.ks;
    const int blocks = gx * gy * ks + b.T + b.E + (b.xdig != nullptr ? b.T : 0);
    void* gargs[] = {&b, &kslice, &gx, &gy, &ks};
    return launch_pdl_raw(fn, dim3(blocks), dim3(kGThreads), smem, stream, gargs);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream, int sms) {
    if (route_tiled_path(a.T, a.H) && a.lsb_x != nullptr && a.part != nullptr) {
        // logits by input slice + row statistics + token digits in one launch; per-token selection
        const RouteTiling r = route_tiling(a.T, a.E, a.H, sms < kRouteMaxSms ? sms : kRouteMaxSms);
        RouteArgs b = a;
        b.ks = r.ks;
        cudaError_t err;
        if (r.TT == 16) err = launch_route_prep<16, 32>(b, r, stream);
        else if (r.TE == 32) err = launch_route_prep<64, 32>(b, r, stream);
        else err = launch_route_prep<64, 128>(b, r, stream);
        if (err != cudaSuccess) return err;
        size_t ssm = (static_cast<size_t>(a.E) * 24 + 15) & ~static_cast<size_t>(15);
        if (ssm > 48 * 1024) {
            err = cudaFuncSetAttribute(route_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(ssm));
            if (err != cudaSuccess) return err;
        }
        void* args[] = {&b};
        return launch_pdl_raw(reinterpret_cast<const void*>(route_select_kernel), dim3(a.T), dim3(a.T <= kSelSmallBatch ? kSelWarpsMax * 32 : 128), ssm, stream,
                              args);
    }
    // few tokens: split each expert's dot product over 4 warps to shorten the serial chain
    RouteArgs b = a;
    b.wpe = a.T <= 16 ? 4 : 1;
    const int epb = kRouteWarps / b.wpe;
    const int chunks = (a.E + epb - 1) / epb;
    size_t smem = static_cast<size_t>(a.H) * 12;              // fp64 token, lowest bits, bf16 copy
    const size_t need_vals = static_cast<size_t>(a.E) * 24;   // logits, keys and exps
    if (need_vals > smem) smem = need_vals;
    smem = (smem + 15) & ~static_cast<size_t>(15);
    const int nq = (a.H / 8 + 32 * b.wpe - 1) / (32 * b.wpe);   // uint4 router loads per lane
    const void* fn = nq <= 2 ? reinterpret_cast<const void*>(route_kernel<2>)
                             : (nq <= 4 ? reinterpret_cast<const void*>(route_kernel<4>)
                                        : reinterpret_cast<const void*>(route_kernel<8>));
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (err != cudaSuccess) return err;
    }
    dim3 grid(chunks, a.T);
    void* args[] = {&b};
    return launch_pdl_raw(fn, grid, dim3(kRouteWarps * 32), smem, stream, args);
}


}  // namespace dpa
