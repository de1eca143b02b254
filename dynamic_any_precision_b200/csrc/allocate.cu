// Post-routing plane allocation and token->expert grouping.
//
// DPA-MoE, Abstract: how many chunks a routed pair reads is decided after routing, from the
// gate scores of the current call. DuoRate, Abstract: per-expert rates trade rate against
// distortion through a Lagrange multiplier, found by bisection. MatMoE, review "Core
// Contribution": a binary search picks the mix of precisions that meets a mean bit-width.
//
// For a multiplier lambda each routed pair p (expert e, gate g) reads
//     k_p(lambda) = argmin_{kmin<=k<=kmax} fl(fl(g * r_e(k)) + fl(lambda * k))
// planes (ties to the smaller k), and N(lambda) = sum_p k_p(lambda). Exactly 64 fp64
// bisection steps on [0, 2*max_p fl(g_p r_e(kmin)) + 1] keep N(hi) <= target * P; the result
// is lambda = hi. Every fp64 operation is an explicitly rounded intrinsic and the file is
// compiled with --fmad=false, so the decisions match any IEEE implementation of these steps.
//
// The 64 sequential steps are evaluated D at a time: the 2^D - 1 midpoints the next D steps
// can visit form a binary tree (a node's interval follows from the steps on its path), every
// node's N(mid) is computed in parallel, and then each thread walks the tree from the root,
// taking at every level exactly the branch the sequential bisection takes. The resulting lo,
// hi and lambda are bit-identical to the step-by-step loop.
//
// Then pairs are grouped by key (expert, k) with a counting sort, and for every expert with
// pairs the kernel writes a work descriptor and a table of two-token tiles (same k) that the
// expert GEMV consumes.
#include <cstdint>

#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kAllocThreads = 1024;       // maximum block size
constexpr int kSmemCostDoubles = 8192;    // costs kept in shared memory up to this many
constexpr int kSmallP = 64;               // up to this many pairs one warp runs the bisection
constexpr int kSpecMaxP = 2048;           // up to this many pairs the whole block speculates and verifies
constexpr int kCoopThreads = 512;         // grid-wide bisection: threads per CTA
constexpr int kCoopMaxPairsPerBlock = 6144;   // shared-memory costs: 6144 pairs x 32 B = 192 KB per CTA
constexpr int kCoopDepth = 6;             // bisection steps per grid round (63 midpoints)
constexpr int kCoopMinPairs = 2048;       // below this the single-CTA bisection is faster
static_assert((64 + kCoopDepth - 1) / kCoopDepth <= kCoopRoundsMax, "round counters");

// The plane counts as fp64 constants, converted once per thread (an integer-to-fp64 conversion
// inside the decision loops costs more than the decision itself), and the candidate loop
// unrolled over the at most four counts (B <= 4).
struct KVals {
    double v[4];
};
__device__ __forceinline__ KVals make_kvals(int kmin) {
    KVals k;
#pragma unroll
    for (int i = 0; i < 4; ++i) k.v[i] = static_cast<double>(kmin + i);
    return k;
}

__device__ __forceinline__ int choose_k(const double* c, int nk, int kmin, const KVals& kv, double lam) {
    double best = __dadd_rn(c[0], __dmul_rn(lam, kv.v[0]));
    int kb = kmin;
#pragma unroll
    for (int i = 1; i < 4; ++i) {
        if (i < nk) {
            const double cost = __dadd_rn(c[i], __dmul_rn(lam, kv.v[i]));
            if (cost < best) { best = cost; kb = kmin + i; }
        }
    }
    return kb;
}

__device__ __forceinline__ double midpoint(double lo, double hi) { return __dmul_rn(0.5, __dadd_rn(lo, hi)); }


// the same decision with the pair's costs in registers
__device__ __forceinline__ int choose_k_reg(const double (&c)[4], int nk, int kmin, const KVals& kv, double lam) {
    double best = __dadd_rn(c[0], __dmul_rn(lam, kv.v[0]));
    int kb = kmin;
#pragma unroll
    for (int i = 1; i < 4; ++i) {
        if (i < nk) {
            const double cost = __dadd_rn(c[i], __dmul_rn(lam, kv.v[i]));
            if (cost < best) { best = cost; kb = kmin + i; }
        }
    }
    return kb;
}

// Stored planes of expert e (per-expert stored widths; else every expert holds kmax).
__device__ __forceinline__ int stored_width(const AllocArgs& a, int e) {
    return a.expert_width ? static_cast<int>(a.expert_width[e]) : a.kmax;
}

constexpr int kRegPairs = 4;   // pairs per lane held in registers by the small-batch bisection
// 1/d for the plane-count gap d = 1..3 of a hull breakpoint (B <= 4); the breakpoints only
// steer the speculation, so a rounded 1/3 is fine
__device__ __forceinline__ double inv_gap(int d) { return d == 1 ? 1.0 : (d == 2 ? 0.5 : 1.0 / 3.0); }

// inclusive block scan of one int per thread
__device__ __forceinline__ int block_incl_scan(int v, int* s_tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) s_tmp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? s_tmp[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        s_tmp[lane] = w;
    }
    __syncthreads();
    const int r = v + (warp > 0 ? s_tmp[warp - 1] : 0);
    __syncthreads();
    return r;
}

// inclusive block scan of NV ints per thread at once (one exchange through shared memory)
template <int NV>
__device__ __forceinline__ void block_incl_scan_n(int (&v)[NV], int (*s_tmp)[32]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int u = __shfl_up_sync(0xffffffffu, v[j], o);
            if (lane >= o) v[j] += u;
        }
    }
    if (lane == 31)
#pragma unroll
        for (int j = 0; j < NV; ++j) s_tmp[j][warp] = v[j];
    __syncthreads();
    if (warp < NV) {   // warp j scans the warp totals of value j
        int w = lane < nw ? s_tmp[warp][lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        s_tmp[warp][lane] = w;
    }
    __syncthreads();
    if (warp > 0)
#pragma unroll
        for (int j = 0; j < NV; ++j) v[j] += s_tmp[j][warp - 1];
    __syncthreads();
}

// Shared-memory carve-up: [costs (if they fit)] [counts E*nk] [seg E*nk+1] [sorted P] [k P]
struct AllocSmem {
    size_t costs, counts, seg, sorted, kk, bp, bj, ptok, rexp, rfirst, total;
    bool costs_in_smem;
};

// recs: the GEMV records are written (token of each grouped position, each record's owner
// expert and each expert's first record are kept in shared memory for them)
__host__ __device__ inline AllocSmem alloc_smem_layout(int P, int E, int nk, bool recs) {
    AllocSmem L;
    L.costs_in_smem = static_cast<size_t>(P) * nk <= static_cast<size_t>(kSmemCostDoubles);
    L.costs = 0;
    size_t off = L.costs_in_smem ? static_cast<size_t>(P) * nk * 8 : 0;
    L.counts = off;
    off += static_cast<size_t>(E) * nk * 4;
    L.seg = off;
    off += (static_cast<size_t>(E) * nk + 1) * 4;
    L.sorted = off;
    off += static_cast<size_t>(P) * 4;
    L.kk = off;
    off += static_cast<size_t>(P);
    // breakpoints of the speculative bisection (mid-size batches): P*(nk-1) doubles and ints
    const size_t nbp = (P > kSmallP && P <= kSpecMaxP && L.costs_in_smem) ? static_cast<size_t>(P) * (nk - 1) : 0;
    off = (off + 7) & ~static_cast<size_t>(7);
    L.bp = off;
    off += nbp * 8;
    L.bj = off;
    off += nbp * 4;
    off = (off + 15) & ~static_cast<size_t>(15);
    const size_t nrec = static_cast<size_t>(P) / 4 + static_cast<size_t>(E) * nk + 1;
    L.ptok = off;
    off += recs ? static_cast<size_t>(P) * 4 : 0;
    L.rexp = off;
    off += recs ? nrec * 4 : 0;
    L.rfirst = off;
    off += recs ? static_cast<size_t>(E) * 4 : 0;
    L.total = (off + 15) & ~static_cast<size_t>(15);
    return L;
}

__global__ void __launch_bounds__(kAllocThreads) allocate_kernel(AllocArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_tmp[32];
    __shared__ int s_scan5[5][32];
    __shared__ double s_max[32];
    __shared__ unsigned char s_pred[2][kAllocThreads];
    // speculative replay of the bisection (small batches)
    __shared__ double s_bp[kSmallP * 3];
    __shared__ int s_bj[kSmallP * 3];
    __shared__ int s_order[kSmallP * 3];
    __shared__ int s_nbp;
    __shared__ double s_mid[64], s_lo[65], s_hi[65];
    __shared__ unsigned char s_spred[64];
    __shared__ unsigned s_mis[8];
    const int P = a.T * a.K;
    const int nk = a.kmax - a.kmin + 1;
    const KVals kv = make_kvals(a.kmin);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const AllocSmem Ls = alloc_smem_layout(P, a.E, nk, a.vrec != nullptr);
    double* c_base = Ls.costs_in_smem ? reinterpret_cast<double*>(smem + Ls.costs) : a.cbuf;
    uint8_t* s_k = smem + Ls.kk;

    // the residual table is static: bring its lines towards this SM while the router finishes
    for (int i = tid * 16; i < a.E * a.B; i += blockDim.x * 16)
        asm volatile("prefetch.global.L1 [%0];" ::"l"(a.rtable + i));
    pdl_wait();   // the routed pairs come from the previous kernel
    pdl_trigger();   // the successor may become resident now (it waits for this kernel)
    // the budget, the pairs' experts and gates are loaded together (one round trip)
    const bool budget_policy = a.policy == DPA_ALLOC_LAGRANGE || a.policy == DPA_ALLOC_UNIFORM;
    const double target = budget_policy ? *a.target : 0.0;   // the other policies read no budget
    const double tau = a.policy == DPA_ALLOC_THRESHOLD ? *a.threshold : 0.0;
    // the budget policies need a target in [kmin, kmax]; the threshold policy a finite threshold
    int bad = a.policy == DPA_ALLOC_THRESHOLD
                  ? ((tau >= -1.0e300 && tau <= 1.0e300) ? 0 : 1)
                  : (!budget_policy || (target >= static_cast<double>(a.kmin) && target <= static_cast<double>(a.kmax)))
                        ? 0 : 1;
    if (bad && tid == 0) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, a.policy == DPA_ALLOC_THRESHOLD ? 12 : 10);
    int bad_e = 0, bad_w = 0;
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = a.idx[p];
        const bool ok = e >= 0 && e < a.E;
        bad_e |= ok ? 0 : 1;
        if (ok && a.expert_width) {
            const int w = a.expert_width[e];
            bad_w |= (w < a.kmin || w > a.kmax) ? 1 : 0;
        }
    }
    const int any_bad_e = __syncthreads_or(bad_e);
    const int any_bad_w = __syncthreads_or(bad_w);
    if (any_bad_e && tid == 0) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 11);
    if (!any_bad_e && any_bad_w && tid == 0) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 15);
    if (bad || any_bad_e || any_bad_w) {
        if (a.do_permute && tid == 0) {   // nothing downstream may read a previous call's work lists
            a.hdr->n_active = 0;
            a.hdr->n_gtiles = 0;
            a.hdr->n_vgroups = 0;
        }
        return;
    }

    if (a.k_given) {   // plane counts (and lambda) already chosen by the grid-wide bisection
        for (int p = tid; p < P; p += blockDim.x) s_k[p] = a.k_out[p];
        __syncthreads();
        goto grouping;
    }
    if (a.policy == DPA_ALLOC_UNIFORM) {
        // equal shares of floor(target * P) planes; the first (budget mod P) pairs one more
        const int nb = static_cast<int>(floor(__dmul_rn(target, static_cast<double>(P))));
        const int base = nb / P, rem = nb - base * P;
        for (int p = tid; p < P; p += blockDim.x) {
            const int k = min(base + (p < rem ? 1 : 0), stored_width(a, a.idx[p]));
            a.k_out[p] = static_cast<uint8_t>(k);
            s_k[p] = static_cast<uint8_t>(k);
        }
        if (tid == 0 && a.lambda_out) *a.lambda_out = 0.0;
        __syncthreads();
        goto grouping;
    }
    if (a.policy == DPA_ALLOC_EXPERT_TABLE) {
        // every pair reads its expert's rate (solved ahead of time from a workload profile)
        int bad_k = 0;
        for (int p = tid; p < P; p += blockDim.x) {
            const int k = a.expert_k[a.idx[p]];
            bad_k |= (k < a.kmin || k > a.kmax) ? 1 : 0;
        }
        if (__syncthreads_or(bad_k)) {
            if (tid == 0) {
                set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 14);
                if (a.do_permute) { a.hdr->n_active = 0; a.hdr->n_gtiles = 0; a.hdr->n_vgroups = 0; }
            }
            return;
        }
        for (int p = tid; p < P; p += blockDim.x) {
            const int k = min(static_cast<int>(a.expert_k[a.idx[p]]), stored_width(a, a.idx[p]));
            a.k_out[p] = static_cast<uint8_t>(k);
            s_k[p] = static_cast<uint8_t>(k);
        }
        if (tid == 0 && a.lambda_out) *a.lambda_out = 0.0;
        __syncthreads();
        goto grouping;
    }
    if (a.policy == DPA_ALLOC_THRESHOLD) {
        // high precision above the calibrated score threshold, low precision otherwise
        for (int p = tid; p < P; p += blockDim.x) {
            const int k = min(a.gate[p] > tau ? a.kmax : a.kmin, stored_width(a, a.idx[p]));
            a.k_out[p] = static_cast<uint8_t>(k);
            s_k[p] = static_cast<uint8_t>(k);
        }
        if (tid == 0 && a.lambda_out) *a.lambda_out = tau;
        __syncthreads();
        goto grouping;
    }
    {
    // costs c[p][i] = fl(g_p * r_{e_p}(kmin + i)); the rtable loads of a pair are issued together
    double mx = 0.0;
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = a.idx[p];
        const double g = a.gate[p];
        const int wmax = stored_width(a, e);   // counts above the expert's stored planes cost +inf
        double r[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < nk) r[i] = a.rtable[static_cast<size_t>(e) * a.B + (a.kmin + i - 1)];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < nk) {
                const double c = a.kmin + i > wmax ? CUDART_INF : __dmul_rn(g, r[i]);
                c_base[static_cast<size_t>(p) * nk + i] = c;
                if (i == 0) mx = fmax(mx, c);
            }
        }
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_max[warp] = mx;
    __syncthreads();
    mx = s_max[0];
    for (int w = 1; w < nw; ++w) mx = fmax(mx, s_max[w]);

    const double budget = __dmul_rn(target, static_cast<double>(P));
    const int nb = static_cast<int>(floor(budget));   // an integer count n exceeds budget iff n > nb
    double lo = 0.0;
    double hi = __dadd_rn(__dmul_rn(2.0, mx), 1.0);

    if (P <= kSmallP) {
        // 8 warps, 4 lanes per node: 64 node slots hold the 63 midpoints of the next 6 steps.
        // Each lane counts planes for every 4th pair; the 4-lane sums give N(mid); each warp's
        // 8 predicates travel through shared memory as one byte, and every thread walks the
        // tree in registers.
        const int slot = tid >> 2, gl = tid & 3;   // node slot 0..31, lane in node
        const double* s_costs = reinterpret_cast<const double*>(smem + Ls.costs);   // P*nk <= kSmemCostDoubles
        // this lane's pairs (gl, gl+4, ...) and their costs, kept in registers across all rounds
        const bool in_regs = P <= 4 * kRegPairs;
        double creg[kRegPairs][4];
#pragma unroll
        for (int j = 0; j < kRegPairs; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int p = gl + 4 * j;
                creg[j][i] = (in_regs && p < P && i < nk) ? s_costs[p * nk + i] : 0.0;
            }
        // ---- speculation. In real arithmetic each pair's choice falls at the breakpoints of the
        // lower convex hull of its points (k, c_k); summing the falls gives the lambda below which
        // N(lambda) > budget. One thread replays the 64 steps with that threshold, recording each
        // midpoint; then every recorded step's predicate is evaluated exactly, in parallel. The
        // replay is kept up to the first step whose exact predicate disagrees; from there the exact
        // tree bisection below takes over. Either way the steps taken are the exact ones.
        if (tid == 0) s_nbp = 0;
        __syncthreads();
        if (tid < P) {
            const double* c = s_costs + tid * nk;
            int cur = 0;   // choice as lambda -> 0+: the smallest cost, ties to the smaller k
            for (int i = 1; i < nk; ++i) if (c[i] < c[cur]) cur = i;
            while (cur > 0) {
                int jn = -1;
                double tn = 0.0;
                for (int j = 0; j < cur; ++j) {   // the next smaller k to take over as lambda grows
                    const double t = __dmul_rn(__dsub_rn(c[j], c[cur]), inv_gap(cur - j));
                    if (jn < 0 || t < tn) { jn = j; tn = t; }
                }
                const int slotb = atomicAdd(&s_nbp, 1);
                s_bp[slotb] = tn;
                s_bj[slotb] = cur - jn;
                cur = jn;
            }
        }
        __syncthreads();
        const int nbp = s_nbp;
        for (int i = tid; i < nbp; i += blockDim.x) {   // descending order of the breakpoints
            const double v = s_bp[i];
            int r = 0;
            for (int j = 0; j < nbp; ++j) r += (s_bp[j] > v || (s_bp[j] == v && j < i)) ? 1 : 0;
            s_order[r] = i;
        }
        __syncthreads();
        if (tid == 0) {
            double lam_c = 0.0;    // N(lambda) > budget exactly for lambda < lam_c (real arithmetic)
            int cum = P * a.kmin;
            for (int m = 0; m < nbp; ++m) {
                cum += s_bj[s_order[m]];
                if (cum > nb) { lam_c = s_bp[s_order[m]]; break; }
            }
            double l = lo, h = hi;
            for (int i = 0; i < 64; ++i) {
                s_lo[i] = l;
                s_hi[i] = h;
                const double m = midpoint(l, h);
                const int pr = m < lam_c ? 1 : 0;
                s_mid[i] = m;
                s_spred[i] = static_cast<unsigned char>(pr);
                if (pr) l = m; else h = m;
            }
            s_lo[64] = l;
            s_hi[64] = h;
        }
        __syncthreads();
        {   // exact check of the 64 recorded steps: four threads per step
            const int node = tid >> 2, gl4 = tid & 3;
            int n = 0;
            const double m = s_mid[node];
            for (int p = gl4; p < P; p += 4) n += choose_k(s_costs + p * nk, nk, a.kmin, kv, m);
            n += __shfl_xor_sync(0xffffffffu, n, 1);
            n += __shfl_xor_sync(0xffffffffu, n, 2);
            const int pr = n > nb ? 1 : 0;
            const unsigned bad_mask = __ballot_sync(0xffffffffu, gl4 == 0 && pr != s_spred[node]);
            if (lane == 0) s_mis[warp] = bad_mask;   // bit 4j of warp w: step 8w + j
        }
        __syncthreads();
        int it0 = 64;
        for (int w = 0; w < 8 && it0 == 64; ++w)
            if (s_mis[w]) it0 = 8 * w + (__ffs(static_cast<int>(s_mis[w])) - 1) / 4;
        lo = s_lo[it0];
        hi = s_hi[it0];

        int round = 0;
        for (int it = it0; it < 64; ++round) {
            const int D = min(6, 64 - it);
            const int node = slot + 1;
            const bool active = node < (1 << D);
            int n = 0;
            if (active) {
                const int depth = 31 - __clz(node);
                double l = lo, h = hi;
                for (int lev = depth - 1; lev >= 0; --lev) {
                    const double m = midpoint(l, h);
                    if ((node >> lev) & 1) l = m; else h = m;
                }
                const double mid = midpoint(l, h);
                if (in_regs) {
#pragma unroll
                    for (int j = 0; j < kRegPairs; ++j)
                        if (gl + 4 * j < P) n += choose_k_reg(creg[j], nk, a.kmin, kv, mid);
                } else {
                    int n0 = 0, n1 = 0;
                    int p = gl;
                    for (; p + 4 < P; p += 8) {   // two independent pairs per iteration
                        n0 += choose_k(s_costs + p * nk, nk, a.kmin, kv, mid);
                        n1 += choose_k(s_costs + (p + 4) * nk, nk, a.kmin, kv, mid);
                    }
                    if (p < P) n0 += choose_k(s_costs + p * nk, nk, a.kmin, kv, mid);
                    n = n0 + n1;
                }
            }
            n += __shfl_xor_sync(0xffffffffu, n, 1);
            n += __shfl_xor_sync(0xffffffffu, n, 2);
            const int pred = (active && n > nb) ? 1 : 0;
            const unsigned bal = __ballot_sync(0xffffffffu, pred && gl == 0);   // bits 4*i: node 8*warp+i+1
            if (lane == 0) {
                unsigned b = 0;
                for (int i = 0; i < 8; ++i) b |= ((bal >> (4 * i)) & 1u) << i;
                s_pred[round & 1][warp] = static_cast<unsigned char>(b);
            }
            __syncthreads();
            unsigned long long mask = 0ull;   // bit node-1
#pragma unroll
            for (int w = 0; w < 8; ++w) mask |= static_cast<unsigned long long>(s_pred[round & 1][w]) << (8 * w);
            int nd = 1;
            for (int lev = 0; lev < D; ++lev) {
                const int pr = static_cast<int>((mask >> (nd - 1)) & 1ull);
                const double m = midpoint(lo, hi);
                if (pr) lo = m; else hi = m;
                nd = 2 * nd + pr;
            }
            it += D;
        }
    } else {
        int it_start = 0;
        if (P <= kSpecMaxP && Ls.costs_in_smem) {
            // ---- speculation for mid-size batches (the same idea as above, at block scale).
            // Breakpoints of every pair's lower convex hull, at fixed slots p*(nk-1)+i (unused: -1).
            const double* s_costs = reinterpret_cast<const double*>(smem + Ls.costs);
            double* s_bpv = reinterpret_cast<double*>(smem + Ls.bp);
            int* s_bjv = reinterpret_cast<int*>(smem + Ls.bj);
            const int nslot = nk - 1;
            for (int p = tid; p < P; p += blockDim.x) {
                const double* c = s_costs + p * nk;
                int cur = 0;
                for (int i = 1; i < nk; ++i) if (c[i] < c[cur]) cur = i;
                int slotb = 0;
                while (cur > 0) {
                    int jn = -1;
                    double tn = 0.0;
                    for (int j = 0; j < cur; ++j) {
                        const double t = __dmul_rn(__dsub_rn(c[j], c[cur]), inv_gap(cur - j));
                        if (jn < 0 || t < tn) { jn = j; tn = t; }
                    }
                    s_bpv[p * nslot + slotb] = tn;
                    s_bjv[p * nslot + slotb] = cur - jn;
                    ++slotb;
                    cur = jn;
                }
                for (; slotb < nslot; ++slotb) {
                    s_bpv[p * nslot + slotb] = -1.0;
                    s_bjv[p * nslot + slotb] = 0;
                }
            }
            // lam_c = the largest breakpoint v with W(>= v) > budget - P*kmin (W: summed jumps):
            // weighted radix select, 8 bits per pass, on the (non-negative) fp64 bit patterns
            __shared__ int s_hist[256];
            __shared__ unsigned long long s_prefix;
            __shared__ double s_rem;
            __shared__ int s_found;
            const int nall = P * nslot;
            if (tid == 0) {
                s_prefix = 0ull;
                s_rem = __dsub_rn(budget, static_cast<double>(P * a.kmin));
                s_found = 1;
            }
            for (int pass = 0; pass < 8; ++pass) {
                const int shift = 56 - 8 * pass;
                for (int b = tid; b < 256; b += blockDim.x) s_hist[b] = 0;
                __syncthreads();
                const unsigned long long pre = s_prefix;
                const unsigned long long hmask = pass == 0 ? 0ull : (~0ull << (shift + 8));
                if (s_found) {
                    // the leading digits repeat across most keys: aggregate equal buckets per warp
                    // before the shared-memory atomic
                    for (int q0 = warp * 32; q0 < nall; q0 += blockDim.x) {
                        const int q = q0 + lane;
                        int bucket = -1, wgt = 0;
                        if (q < nall) {
                            const double v = s_bpv[q];
                            if (v >= 0.0) {
                                const unsigned long long key = static_cast<unsigned long long>(__double_as_longlong(v));
                                if ((key & hmask) == pre) {
                                    bucket = static_cast<int>((key >> shift) & 255u);
                                    wgt = s_bjv[q];
                                }
                            }
                        }
                        const unsigned grp = __match_any_sync(0xffffffffu, bucket);
                        const int tot = static_cast<int>(__reduce_add_sync(grp, static_cast<unsigned>(wgt)));
                        if (bucket >= 0 && lane == __ffs(static_cast<int>(grp)) - 1) atomicAdd(&s_hist[bucket], tot);
                    }
                }
                __syncthreads();
                if (warp == 0 && s_found) {
                    // lane l holds buckets 255-8l .. 248-8l; the first bucket from the top whose
                    // cumulative weight exceeds the remainder is picked
                    const double rem = s_rem;
                    int part = 0;
                    for (int u = 0; u < 8; ++u) part += s_hist[255 - 8 * lane - u];
                    int incl = part;
                    for (int o = 1; o < 32; o <<= 1) {
                        const int t = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += t;
                    }
                    const int excl = incl - part;
                    const bool crosses = static_cast<double>(incl) > rem && !(static_cast<double>(excl) > rem);
                    const unsigned who = __ballot_sync(0xffffffffu, crosses);
                    if (who == 0u) {
                        if (lane == 0) s_found = 0;   // the jumps never exceed the budget: lam_c = 0
                    } else if (lane == __ffs(static_cast<int>(who)) - 1) {
                        int acc = excl, pick = -1;
                        for (int u = 0; u < 8; ++u) {
                            const int b = 255 - 8 * lane - u;
                            const int h = s_hist[b];
                            if (static_cast<double>(acc + h) > rem) { pick = b; break; }
                            acc += h;
                        }
                        s_prefix = pre | (static_cast<unsigned long long>(pick) << shift);
                        s_rem = __dsub_rn(rem, static_cast<double>(acc));
                    }
                }
                __syncthreads();
            }
            if (tid == 0) {
                const double lam_c = s_found ? __longlong_as_double(static_cast<long long>(s_prefix)) : 0.0;
                double l = lo, h = hi;
                for (int i = 0; i < 64; ++i) {   // replay with the real-arithmetic predicate
                    s_lo[i] = l;
                    s_hi[i] = h;
                    const double m = midpoint(l, h);
                    const int pr = m < lam_c ? 1 : 0;
                    s_mid[i] = m;
                    s_spred[i] = static_cast<unsigned char>(pr);
                    if (pr) l = m; else h = m;
                }
                s_lo[64] = l;
                s_hi[64] = h;
            }
            __syncthreads();
            // exact check of the 64 recorded steps: warp w checks steps 2w and 2w+1 (32 warps)
            for (int st0 = 2 * warp; st0 < 64; st0 += 2 * nw) {
                const double m0 = s_mid[st0], m1 = s_mid[st0 + 1];
                int n0 = 0, n1 = 0;
                for (int p = lane; p < P; p += 32) {
                    const double* c = s_costs + p * nk;
                    n0 += choose_k(c, nk, a.kmin, kv, m0);
                    n1 += choose_k(c, nk, a.kmin, kv, m1);
                }
                n0 = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(n0)));
                n1 = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(n1)));
                if (lane == 0) {
                    s_pred[0][st0] = (n0 > nb ? 1 : 0) != s_spred[st0] ? 1 : 0;
                    s_pred[0][st0 + 1] = (n1 > nb ? 1 : 0) != s_spred[st0 + 1] ? 1 : 0;
                }
            }
            __syncthreads();
            int it0 = 64;
            for (int i = 0; i < 64; ++i)
                if (s_pred[0][i]) { it0 = i; break; }
            lo = s_lo[it0];
            hi = s_hi[it0];
            it_start = it0;
            __syncthreads();   // s_pred is reused by the tree below
        }
        // whole block: a group of gs threads per node, trees of depth D per round
        int gs_log = 0;
        while ((1 << gs_log) < 32 && (P >> (gs_log + 3)) > 0) ++gs_log;   // ~8 pairs per thread
        const int gs = 1 << gs_log;
        int lg_threads = 31 - __clz(blockDim.x);
        int dmax = lg_threads - gs_log;
        if (dmax > 7) dmax = 7;
        const int node_slot = tid >> gs_log;
        const int glane = tid & (gs - 1);
        int round = 0;
        for (int it = it_start; it < 64; ++round) {
            const int D = min(dmax, 64 - it);
            const int n_nodes = (1 << D) - 1;
            const int node = node_slot + 1;   // heap index
            const bool active = node_slot < n_nodes;
            int local = 0;
            if (active) {
                const int depth = 31 - __clz(node);
                double l = lo, h = hi;
                for (int lev = depth - 1; lev >= 0; --lev) {
                    const double m = midpoint(l, h);
                    if ((node >> lev) & 1) l = m; else h = m;
                }
                const double mid = midpoint(l, h);
                for (int p = glane; p < P; p += gs) local += choose_k(c_base + static_cast<size_t>(p) * nk, nk, a.kmin, kv, mid);
            }
            // every lane of the warp takes part in the group reduction (inactive lanes add 0)
            for (int o = gs >> 1; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
            if (active && glane == 0) s_pred[round & 1][node] = local > nb ? 1 : 0;
            __syncthreads();
            int node_w = 1;
            for (int lev = 0; lev < D; ++lev) {
                const int pr = s_pred[round & 1][node_w];
                const double m = midpoint(lo, hi);
                if (pr) lo = m; else hi = m;
                node_w = 2 * node_w + pr;
            }
            it += D;
        }
    }
    // final plane counts
    for (int p = tid; p < P; p += blockDim.x) {
        const int k = choose_k(c_base + static_cast<size_t>(p) * nk, nk, a.kmin, kv, hi);
        a.k_out[p] = static_cast<uint8_t>(k);
        s_k[p] = static_cast<uint8_t>(k);
    }
    if (tid == 0 && a.lambda_out) *a.lambda_out = hi;
    }
grouping:
    if (!a.do_permute) return;

    // ---------------- grouping by (expert, k), all in shared memory ----------------
    int* s_counts = reinterpret_cast<int*>(smem + Ls.counts);
    int* s_seg = reinterpret_cast<int*>(smem + Ls.seg);
    int* s_sorted = reinterpret_cast<int*>(smem + Ls.sorted);
    const int nkeys = a.E * nk;
    for (int i = tid; i < nkeys; i += blockDim.x) s_counts[i] = 0;
    __syncthreads();
    for (int p = tid; p < P; p += blockDim.x) atomicAdd(&s_counts[a.idx[p] * nk + (s_k[p] - a.kmin)], 1);
    __syncthreads();
    {   // exclusive scan of the counts into s_seg; counts become placement cursors
        const int per = (nkeys + blockDim.x - 1) / blockDim.x;
        const int k0 = tid * per, k1 = min(nkeys, k0 + per);
        int run = 0;
        for (int i = k0; i < k1; ++i) run += s_counts[i];
        int base = block_incl_scan(run, s_tmp) - run;
        for (int i = k0; i < k1; ++i) {
            const int c = s_counts[i];
            s_seg[i] = base;
            s_counts[i] = base;
            base += c;
        }
        if (tid == 0) s_seg[nkeys] = P;
    }
    __syncthreads();
    int* s_ptok = reinterpret_cast<int*>(smem + Ls.ptok);   // token of each grouped position
    for (int p = tid; p < P; p += blockDim.x) {
        const int key = a.idx[p] * nk + (s_k[p] - a.kmin);
        const int pos = atomicAdd(&s_counts[key], 1);
        const int tok = p / a.K;
        s_sorted[pos] = p;
        if (a.vrec) s_ptok[pos] = tok;
        a.pair_pos[p] = pos;
        if (a.pos_tok) a.pos_tok[pos] = tok;
    }
    __syncthreads();
    // Per expert: the prefill GEMM's token tiles (one (expert, k) class each) and the start of its
    // GEMV records (groups of up to vtpg tiles of up to 4 pairs of one class, classes ascending in
    // k); experts in rounds of blockDim so that both lists stay in ascending expert order. Each
    // record's owner expert goes to s_rexp; the records themselves are written below, one warp
    // per record.
    int rank_base = 0, gt_base = 0, vg_base = 0;
    const int vtpg = a.vtiles_per_group > 0 ? a.vtiles_per_group : 1;
    int* s_rexp = reinterpret_cast<int*>(smem + Ls.rexp);   // [records] owner expert
    int* s_rfirst = reinterpret_cast<int*>(smem + Ls.rfirst);   // [E] first record of each expert
    for (int e0 = 0; e0 < a.E; e0 += blockDim.x) {
        const int e = e0 + tid;
        int km = 0, ngt = 0, nvt = 0;
        if (e < a.E) {
            for (int i = 0; i < nk; ++i) {
                const int n = s_seg[e * nk + i + 1] - s_seg[e * nk + i];
                if (n > 0) km = a.kmin + i;
                ngt += (n + kGemmTileTokens - 1) / kGemmTileTokens;
                nvt += (n + 3) >> 2;
            }
        }
        const int nvg = a.vrec ? (nvt + vtpg - 1) / vtpg : 0;
        const int flag = km > 0 ? 1 : 0;
        int sc[3] = {flag, a.gtiles ? ngt : 0, nvg};   // one block scan of the three counts
        block_incl_scan_n<3>(sc, s_scan5);
        if (a.gtiles && ngt > 0) {   // token tiles of the prefill GEMMs: one (expert, k) class each
            int t = gt_base + sc[1] - ngt;
            for (int i = 0; i < nk; ++i) {
                const int s0 = s_seg[e * nk + i];
                const int n = s_seg[e * nk + i + 1] - s0;
                for (int j = 0; j < n; j += kGemmTileTokens)
                    a.gtiles[t++] = make_int4(e, a.kmin + i, s0 + j, min(kGemmTileTokens, n - j));
            }
        }
        if (a.vrec && e < a.E) {
            const int r0 = vg_base + sc[2] - nvg;
            s_rfirst[e] = r0;
            for (int j = 0; j < nvg; ++j) s_rexp[r0 + j] = e;
        }
        // totals of this round: the scan's last warp totals, still in shared memory; every thread
        // reads them before the barrier below, ahead of the next round's scan
        rank_base += s_scan5[0][nw - 1];
        gt_base += s_scan5[1][nw - 1];
        vg_base += s_scan5[2][nw - 1];
        __syncthreads();
    }
    if (a.vrec) {
        // record r of expert e holds the expert's tiles [j vtpg, (j+1) vtpg), j = r - first(e);
        // lane q computes field q (layout of kVRecInts) and the warp stores the record at once
        for (int r = warp; r < vg_base; r += nw) {
            const int e = s_rexp[r];
            const int j = r - s_rfirst[e];
            int tk[2] = {0, 0}, tn[2] = {0, 0}, tpos[2] = {0, 0}, nt = 0;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                int g = j * vtpg + t;   // the expert's tile index
                if (t >= vtpg) break;
                for (int i = 0; i < nk; ++i) {
                    const int s0 = s_seg[e * nk + i];
                    const int n = s_seg[e * nk + i + 1] - s0;
                    const int ntc = (n + 3) >> 2;
                    if (g < ntc) {
                        tk[t] = a.kmin + i;
                        tn[t] = min(4, n - 4 * g);
                        tpos[t] = s0 + 4 * g;
                        nt = t + 1;
                        break;
                    }
                    g -= ntc;
                }
            }
            int v = 0;
            if (lane == 0) v = e;
            else if (lane == 1) v = tk[nt - 1];            // tiles ascend in k: the last is the group's kmax
            else if (lane == 2) v = nt;
            else if (lane == 4 || lane == 5) v = tk[lane - 4];
            else if (lane == 6 || lane == 7) v = tn[lane - 6];
            else if (lane >= 8 && lane < 24) {
                const int f = lane & 7, t = f >> 2, u = f & 3;
                const bool used = t < nt && u < tn[t];
                v = !used ? -1 : (lane < 16 ? tpos[t] + u : s_ptok[tpos[t] + u]);
            }
            a.vrec[static_cast<size_t>(r) * kVRecInts + lane] = v;
            // the record's work weight per row block (planes read, token tiles), in the owner slot
            __syncwarp();
            if (lane == 0) s_rexp[r] = 5 + 2 * tk[nt - 1] + 3 * nt;
        }
        const bool tab0 = a.vstart[0] && vg_base * a.vnrb[0] > a.vgrid[0];
        const bool tab1 = a.vstart[1] && vg_base * a.vnrb[1] > a.vgrid[1];
        if (tab0 || tab1) {   // (with no more items than CTAs the GEMV splits items evenly)
            __syncthreads();
            // exclusive prefix of the weights over the records: s_rexp[0..vg_base]
            const int nrec = vg_base;
            const int per = (nrec + blockDim.x - 1) / blockDim.x;
            const int r0 = tid * per, r1 = min(nrec, r0 + per);
            int run = 0;
            for (int r = r0; r < r1; ++r) run += s_rexp[r];
            int base = block_incl_scan(run, s_tmp) - run;
            for (int r = r0; r < r1; ++r) {
                const int w = s_rexp[r];
                s_rexp[r] = base;
                base += w;
            }
            if (tid == blockDim.x - 1) s_rexp[nrec] = base;   // the total (the last thread's running sum)
            __syncthreads();
            const long long wtot = s_rexp[nrec];
            for (int j = 0; j < 2; ++j) {
                if (!(j == 0 ? tab0 : tab1)) continue;
                const int grid = a.vgrid[j], nrb = a.vnrb[j];
                for (int b = tid; b <= grid; b += blockDim.x) {
                    // first item i whose preceding work reaches b/grid of the total
                    const long long tb = wtot * nrb * b / grid;
                    int lo = 0, hi = nrec;   // largest g with prefix(g) * nrb <= tb
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (static_cast<long long>(s_rexp[mid]) * nrb <= tb) lo = mid;
                        else hi = mid - 1;
                    }
                    long long start;
                    if (lo >= nrec) {
                        start = static_cast<long long>(nrec) * nrb;
                    } else {
                        const long long pg = static_cast<long long>(s_rexp[lo]) * nrb;
                        const long long wg = s_rexp[lo + 1] - s_rexp[lo];
                        long long rb = (tb - pg + wg - 1) / wg;
                        if (rb > nrb) rb = nrb;
                        start = static_cast<long long>(lo) * nrb + rb;
                    }
                    a.vstart[j][b] = static_cast<int32_t>(start);
                }
            }
        }
    }
    if (tid == 0) {
        a.hdr->n_active = static_cast<uint32_t>(rank_base);
        a.hdr->n_gtiles = static_cast<uint32_t>(gt_base);
        a.hdr->n_vgroups = static_cast<uint32_t>(vg_base);
    }
}

// ---------------- grid-wide bisection for large batches ----------------
// The same 64 exact steps, evaluated by every SM: each CTA keeps the costs of its share of the
// pairs in shared memory; a round computes N(mid) for the 2^D - 1 midpoints the next D
// steps can visit (integer sums, so the order of the additions does not matter), a bounded
// grid barrier publishes the counts, and every thread walks the tree with the exact predicates.

__global__ void __launch_bounds__(kCoopThreads) allocate_coop_kernel(AllocArgs a, CoopSync* cs, int per_block) {
    // this CTA's pairs [p0, p1) with their costs in shared memory; warp w evaluates the
    // midpoints w+1, w+1+nw, ... over all of them (lanes stride the pairs)
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double* s_c = reinterpret_cast<double*>(smem_raw);   // [per_block][4]
    __shared__ double s_mid[64];
    __shared__ double s_red[kCoopThreads / 32];
    __shared__ int s_flag;
    const int P = a.T * a.K;
    const int nk = a.kmax - a.kmin + 1;
    const KVals kv = make_kvals(a.kmin);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const unsigned G = gridDim.x;
    const int p0 = blockIdx.x * per_block, p1 = min(P, p0 + per_block), np = max(0, p1 - p0);

    const double target = *a.target;
    if (!(target >= static_cast<double>(a.kmin) && target <= static_cast<double>(a.kmax))) {
        if (blockIdx.x == 0 && tid == 0) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 10);
        return;   // every CTA reads the same target: the whole grid leaves here
    }
    double mx = 0.0;
    int bad_e = 0;
    for (int j = tid; j < np; j += blockDim.x) {
        const int p = p0 + j;
        const int e = a.idx[p];
        double c[4] = {0.0, 0.0, 0.0, 0.0};
        if (e < 0 || e >= a.E || (a.expert_width && (a.expert_width[e] < a.kmin || a.expert_width[e] > a.kmax))) {
            bad_e = 1;
        } else {
            const double g = a.gate[p];
            const int wmax = stored_width(a, e);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i < nk)
                    c[i] = a.kmin + i > wmax ? CUDART_INF
                                             : __dmul_rn(g, a.rtable[static_cast<size_t>(e) * a.B + (a.kmin + i - 1)]);
            mx = fmax(mx, c[0]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) s_c[4 * j + i] = c[i];
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_red[warp] = mx;
    const int any_bad = __syncthreads_or(bad_e);
    if (tid == 0) {
        double m = s_red[0];
        for (int w = 1; w < nw; ++w) m = fmax(m, s_red[w]);
        // costs are >= 0, so their bit patterns order like their values
        atomicMax(&cs->mx_bits, static_cast<unsigned long long>(__double_as_longlong(m)));
        if (any_bad) atomicOr(&cs->bad, 1u);
    }
    unsigned phase = 1;
    if (!grid_barrier(&cs->barrier, G * phase++, a.hdr, &s_flag)) return;
    if (__ldcg(&cs->bad)) {
        if (blockIdx.x == 0 && tid == 0) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 11);
        return;
    }
    mx = __longlong_as_double(static_cast<long long>(__ldcg(&cs->mx_bits)));
    const double budget = __dmul_rn(target, static_cast<double>(P));
    const int nb = static_cast<int>(floor(budget));   // an integer count n exceeds budget iff n > nb
    double lo = 0.0;
    double hi = __dadd_rn(__dmul_rn(2.0, mx), 1.0);

    int round = 0;
    for (int it = 0; it < 64; ++round) {
        const int D = min(kCoopDepth, 64 - it);
        const int n_nodes = (1 << D) - 1;
        if (tid < n_nodes) {   // midpoint of heap node tid + 1: replay its path from the root
            const int node = tid + 1;
            const int depth = 31 - __clz(node);
            double l = lo, h = hi;
            for (int lev = depth - 1; lev >= 0; --lev) {
                const double m = midpoint(l, h);
                if ((node >> lev) & 1) l = m; else h = m;
            }
            s_mid[node] = midpoint(l, h);
        }
        __syncthreads();
        for (int node = warp + 1; node <= n_nodes; node += nw) {
            const double m = s_mid[node];
            int n = 0;
            for (int j = lane; j < np; j += 32) {
                n += choose_k(s_c + 4 * j, nk, a.kmin, kv, m);
            }
            n = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(n)));
            if (lane == 0 && n) atomicAdd(&cs->counts[round][node][0], n);
        }
        if (!grid_barrier(&cs->barrier, G * phase++, a.hdr, &s_flag)) return;
        int nd = 1;
        for (int lev = 0; lev < D; ++lev) {
            const int n = __ldcg(&cs->counts[round][nd][0]);
            const int pr = n > nb ? 1 : 0;
            const double m = midpoint(lo, hi);
            if (pr) lo = m; else hi = m;
            nd = 2 * nd + pr;
        }
        it += D;
    }
    for (int j = tid; j < np; j += blockDim.x) {
        a.k_out[p0 + j] = static_cast<uint8_t>(choose_k(s_c + 4 * j, nk, a.kmin, kv, hi));
    }
    if (blockIdx.x == 0 && tid == 0 && a.lambda_out) *a.lambda_out = hi;
}

// ---------------- threshold calibration (score-threshold policy) ----------------
// MatMoE, review "Core Contribution": a binary search over a calibration distribution of routing
// scores sets the threshold above which an expert runs at high precision, so that the average
// bit-width meets the target. 64 fp64 bisection steps on [0, 1]: with c(mid) = #{s > mid},
// the plane count kmin*n + (kmax-kmin)*c(mid) above floor(target*n) moves lo up, else hi down;
// the threshold is hi. One CTA; the counts are exact integer sums.
constexpr int kCalibThreads = 1024;

__global__ void __launch_bounds__(kCalibThreads) calibrate_kernel(CalibArgs a) {
    __shared__ int s_cnt[kCalibThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    pdl_wait();
    const double target = *a.target;
    if (!(target >= static_cast<double>(a.kmin) && target <= static_cast<double>(a.kmax))) {
        if (tid == 0) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 13);
        return;
    }
    const long long nb = static_cast<long long>(floor(__dmul_rn(target, static_cast<double>(a.n))));
    const long long base = static_cast<long long>(a.kmin) * a.n;
    const int dk = a.kmax - a.kmin;
    double lo = 0.0, hi = 1.0;
    for (int it = 0; it < 64; ++it) {
        const double mid = __dmul_rn(0.5, __dadd_rn(lo, hi));
        int c = 0;
        for (int i = tid; i < a.n; i += blockDim.x) c += a.scores[i] > mid ? 1 : 0;
        c = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c)));
        if (lane == 0) s_cnt[warp] = c;
        __syncthreads();
        long long tot = 0;
        for (int w = 0; w < nw; ++w) tot += s_cnt[w];
        __syncthreads();
        if (base + static_cast<long long>(dk) * tot > nb) lo = mid; else hi = mid;
    }
    if (tid == 0) *a.threshold_out = hi;
}

}  // namespace

cudaError_t launch_calibrate(const CalibArgs& a, cudaStream_t stream) {
    CalibArgs b = a;
    void* args[] = {&b};
    return launch_pdl_raw(reinterpret_cast<const void*>(calibrate_kernel), dim3(1), dim3(kCalibThreads), 0, stream,
                          args);
}

size_t allocate_smem_bytes(int P, int E, int nk, bool recs) { return alloc_smem_layout(P, E, nk, recs).total; }

int allocate_threads(int P) { return P <= kSmallP ? 256 : kAllocThreads; }   // small: 8 warps x 8 nodes

cudaError_t launch_allocate(const AllocArgs& a, cudaStream_t stream, CoopSync* coop, int sms) {
    const int nk = a.kmax - a.kmin + 1;
    const int P = a.T * a.K;
    AllocArgs b = a;
    const int coop_blocks = sms > 0 ? (P / 64 < sms ? (P + 63) / 64 : sms) : 1;
    int per_block = (P + coop_blocks - 1) / coop_blocks;
    if (coop && a.policy == DPA_ALLOC_LAGRANGE && P > kCoopMinPairs && per_block <= kCoopMaxPairsPerBlock) {
        // grid-wide bisection: the pairs split over (at most) every SM, costs in shared memory
        const int blocks = coop_blocks;
        const size_t smem = static_cast<size_t>(per_block) * 32;
        cudaError_t err = cudaMemsetAsync(coop, 0, sizeof(CoopSync), stream);
        if (err != cudaSuccess) return err;
        if (smem > 48 * 1024) {
            err = cudaFuncSetAttribute(allocate_coop_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
            if (err != cudaSuccess) return err;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(blocks);
        cfg.blockDim = dim3(kCoopThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        void* cargs[] = {&b, &coop, &per_block};
        err = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(allocate_coop_kernel), cargs);
        if (err != cudaSuccess) return err;
        b.k_given = 1;
    }
    const size_t smem = allocate_smem_bytes(P, a.E, nk, a.vrec != nullptr);
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(allocate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
        if (err != cudaSuccess) return err;
    }
    void* args[] = {&b};
    return launch_pdl_raw(reinterpret_cast<const void*>(allocate_kernel), dim3(1), dim3(allocate_threads(P)), smem,
                          stream, args);
}

}  // namespace dpa
