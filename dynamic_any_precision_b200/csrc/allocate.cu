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
// Where the steps run: up to 64 pairs one CTA, speculating (a replay against the summed hull
// breakpoints, checked exactly, trees from the first disagreement); 65 to 2048 pairs a cluster of
// 16 CTAs that split each tree's nodes and exchange the nodes' predicates through distributed
// shared memory, evaluating after one pruning pass only the pairs whose choice can still change;
// beyond, every SM (cooperative launch, grid barrier per tree).
//
// Then pairs are grouped by key (expert, k) with a counting sort; per expert the prefill GEMM's
// token tiles and the expert GEMV's token-group records, and for the two GEMV launches the
// work-balanced ranges of their CTAs.
#include <cstdint>

#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kAllocThreads = 1024;       // maximum block size
constexpr int kSmemCostDoubles = 8192;    // costs kept in shared memory up to this many
constexpr int kSmallP = 64;               // up to this many pairs one warp runs the bisection
constexpr int kSpecMaxP = 2048;           // up to this many pairs (Lagrangian): the cluster bisection
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
    size_t costs, counts, seg, sorted, kk, ptok, rexp, rfirst, total;
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

// Grouping of the pairs by (expert, k) once every pair's plane count is in s_k (this CTA's
// shared memory, P entries): positions, the prefill GEMM's token tiles, the GEMV records and
// the GEMV launches' work-balanced CTA ranges. Whole block.
__device__ void group_pairs(const AllocArgs& a, unsigned char* smem, const AllocSmem& Ls, int P, int nk,
                            const uint8_t* s_k, int* s_tmp, int (*s_scan5)[32]) {
    const int tid = threadIdx.x, nw = blockDim.x >> 5;

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
    // Per expert: the prefill GEMM's token tiles (one (expert, k) class each) and its GEMV records
    // (groups of up to vtpg tiles of up to 4 pairs of one class, classes ascending in k); experts
    // in rounds of blockDim so that both lists stay in ascending expert order. Each record's work
    // weight goes to s_rexp for the balanced ranges below.
    int rank_base = 0, gt_base = 0, vg_base = 0;
    const int vtpg = a.vtiles_per_group > 0 ? a.vtiles_per_group : 1;
    int* s_rexp = reinterpret_cast<int*>(smem + Ls.rexp);   // [records] work weight, then its prefix
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
        if (a.vrec && nvg > 0) {
            // this expert's records: its tiles in class order, vtpg per record, each record of
            // kVRecInts ints written as eight 16-byte stores; its work weight to s_rexp[r]
            int r = vg_base + sc[2] - nvg;
            int t = 0, kk0 = 0, nn0 = 0, qq0 = 0, kk1 = 0, nn1 = 0, qq1 = 0;
            for (int i = 0; i < nk; ++i) {
                const int s0 = s_seg[e * nk + i];
                const int n = s_seg[e * nk + i + 1] - s0;
                for (int j = 0; j < n; j += 4) {
                    if (t == 0) { kk0 = a.kmin + i; nn0 = min(4, n - j); qq0 = s0 + j; }
                    else { kk1 = a.kmin + i; nn1 = min(4, n - j); qq1 = s0 + j; }
                    ++t;
                    const bool last = j + 4 >= n && i == nk - 1;
                    bool more = false;   // any tile of a later class?
                    if (j + 4 >= n)
                        for (int i2 = i + 1; i2 < nk; ++i2) more |= s_seg[e * nk + i2 + 1] > s_seg[e * nk + i2];
                    if (t == vtpg || (j + 4 >= n && !more) || last) {
                        const int nt = t, klast = nt == 2 ? kk1 : kk0;
                        int4* dst = reinterpret_cast<int4*>(a.vrec + static_cast<size_t>(r) * kVRecInts);
                        auto pos = [&](int tt, int u) {
                            const int nn = tt == 0 ? nn0 : (nt == 2 ? nn1 : 0);
                            return u < nn ? (tt == 0 ? qq0 : qq1) + u : -1;
                        };
                        auto tok = [&](int tt, int u) {
                            const int p = pos(tt, u);
                            return p < 0 ? -1 : s_ptok[p];
                        };
                        dst[0] = make_int4(e, klast, nt, 0);
                        dst[1] = make_int4(kk0, nt == 2 ? kk1 : 0, nn0, nt == 2 ? nn1 : 0);
                        dst[2] = make_int4(pos(0, 0), pos(0, 1), pos(0, 2), pos(0, 3));
                        dst[3] = make_int4(pos(1, 0), pos(1, 1), pos(1, 2), pos(1, 3));
                        dst[4] = make_int4(tok(0, 0), tok(0, 1), tok(0, 2), tok(0, 3));
                        dst[5] = make_int4(tok(1, 0), tok(1, 1), tok(1, 2), tok(1, 3));
                        dst[6] = make_int4(0, 0, 0, 0);
                        dst[7] = make_int4(0, 0, 0, 0);
                        s_rexp[r] = 5 + 2 * klast + 3 * nt;   // work weight per row block
                        ++r;
                        t = 0;
                    }
                }
            }
        }
        // totals of this round: the scan's last warp totals, still in shared memory; every thread
        // reads them before the barrier below, ahead of the next round's scan
        rank_base += s_scan5[0][nw - 1];
        gt_base += s_scan5[1][nw - 1];
        vg_base += s_scan5[2][nw - 1];
        __syncthreads();
    }
    if (a.vrec) {
        const bool tab0 = a.vstart[0] && vg_base * a.vnrb[0] > 2 * a.vgrid[0];
        const bool tab1 = a.vstart[1] && vg_base * a.vnrb[1] > 2 * a.vgrid[1];
        if (tab0 || tab1) {   // (with at most two items per CTA the GEMV splits items evenly)
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
        const int it_start = 0;   // (65 to 2048 pairs run on the cluster kernel; this is the general tree)
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
    group_pairs(a, smem, Ls, P, nk, s_k, s_tmp, s_scan5);

}

// ---------------- cluster bisection for mid-size batches ----------------
// The same 64 exact steps, run by a cluster of kClCtas CTAs (one per SM), every CTA holding all
// P pairs' costs in shared memory. A round takes D steps: the 2^D - 1 midpoints those steps can
// visit form a tree (heap order). Node n belongs to CTA (n - 1) mod kClCtas; each of a CTA's
// nodes is one warp, which computes the node's midpoint, counts planes over the listed pairs,
// and stores the node's predicate into every CTA's shared memory with st.async, completing on
// that CTA's round barrier (armed with the bytes it expects; waits bounded). Then every thread
// walks the D steps with the predicates, recomputing the path's midpoints. One block barrier
// per round.
// Pruning, once, at the start of round kClPruneRound. A pair's cost of a count,
// v_k(lam) = fl(c_k + fl(lam k)), never decreases as lam grows (both roundings are monotone).
// So if, a being the pair's choice at hi, v_a(hi) < v_b(lo) for every count b below a and
// v_a(hi) <= v_b(lo) for every count above a (the first minimum wins ties), the pair chooses a
// everywhere in [lo, hi] and so at every later midpoint (they all lie in [lo, hi]): its count
// joins a fixed sum and it leaves the list the nodes evaluate. After the first rounds only pairs
// with a breakpoint near the final lambda stay listed.
#ifndef DPA_ALLOC_CLUSTER
#define DPA_ALLOC_CLUSTER 16
#endif
constexpr int kClCtas = DPA_ALLOC_CLUSTER;      // CTAs of the cluster (16: a non-portable cluster size)
constexpr int kClThreads = 512;
constexpr int kClWarps = kClThreads / 32;
#ifndef DPA_ALLOC_CL_DEPTH_EARLY
#define DPA_ALLOC_CL_DEPTH_EARLY 6
#endif
constexpr int kClDepthEarly = DPA_ALLOC_CL_DEPTH_EARLY;   // steps of the rounds before the pruning (every pair listed)
constexpr int kClDepth = 8;                     // steps of the later rounds
constexpr int kClPruneRound = 2;
constexpr int kClNodes = 1 << kClDepth;
constexpr int kClNodesPerCta = (kClNodes - 1 + kClCtas - 1) / kClCtas;
constexpr int kClMinPairs = 65;                 // below: the single-CTA kernel's small-batch path
static_assert((kClCtas & (kClCtas - 1)) == 0, "cluster size a power of two");
static_assert(kClNodesPerCta <= kClWarps, "at least one warp per node");
static_assert(kClCtas <= 32, "one lane per destination CTA");

// Predicates are kept for three rounds: a warp that owns no node may still be walking round r
// when the other CTAs send round r + 2 (their round r + 1 needs only this CTA's node warps), but
// round r + 3 needs this CTA past its round r + 1 barrier, which every warp reaches after its
// round r walk. The barriers alternate by parity: a round's stores into a barrier can start only
// after this CTA has waited on the round two before.
struct ClShared {
    uint64_t rbar[2];                          // a round's predicates have arrived (by round parity)
    int pw[3][kClNodes];                       // node predicates [round mod 3][heap index]
};

__global__ void __launch_bounds__(kClThreads, 1) allocate_cluster_kernel(AllocArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ ClShared cs;
    __shared__ int s_tmp[32];
    __shared__ int s_scan5[5][32];
    __shared__ double s_wmx[kClWarps];
    __shared__ int s_part[kClNodesPerCta];   // plane counts of nodes shared by several warps
    __shared__ int s_nl;       // listed pairs
    __shared__ int s_fixed;    // planes of the pairs that left the list
    __shared__ int s_bad;
    const int P = a.T * a.K;
    const int nk = a.kmax - a.kmin + 1;
    const KVals kv = make_kvals(a.kmin);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rank = static_cast<int>(cluster_ctarank());
    const AllocSmem Ls = alloc_smem_layout(P, a.E, nk, a.vrec != nullptr);
    double* s_c = reinterpret_cast<double*>(smem + Ls.total);                    // [P][nk] costs
    int* s_list = reinterpret_cast<int*>(s_c + static_cast<size_t>(P) * nk);    // [P] listed pairs
    uint8_t* s_kf = reinterpret_cast<uint8_t*>(s_list + P);                     // [P] final counts
    uint8_t* s_k = smem + Ls.kk;
    if (tid == 0) {
        mbar_init(&cs.rbar[0], 1);
        mbar_init(&cs.rbar[1], 1);
        s_nl = P;
        s_fixed = 0;
        s_bad = 0;
        fence_mbarrier_init_cluster();
    }
    for (int i = tid * 16; i < a.E * a.B; i += blockDim.x * 16)
        asm volatile("prefetch.global.L1 [%0];" ::"l"(a.rtable + i));
    cluster_barrier_once();   // every CTA's barriers exist before anyone stores into it
    pdl_wait();
    pdl_trigger();
    // ---- inputs, checked by every CTA alike (so all take the same exit): budget, expert ids,
    // stored widths; every pair's costs
    const double target = *a.target;
    int flags = (target >= static_cast<double>(a.kmin) && target <= static_cast<double>(a.kmax)) ? 0 : 1;
    double mx = 0.0;
    for (int p = tid; p < P; p += blockDim.x) {
        s_list[p] = p;
        const int e = a.idx[p];
        if (e < 0 || e >= a.E) {
            flags |= 2;
            continue;
        }
        const int wmax = stored_width(a, e);
        if (wmax < a.kmin || wmax > a.kmax) {
            flags |= 4;
            continue;
        }
        const double g = a.gate[p];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i < nk) {
                const double c = a.kmin + i > wmax ? CUDART_INF
                                                   : __dmul_rn(g, a.rtable[static_cast<size_t>(e) * a.B + (a.kmin + i - 1)]);
                s_c[p * nk + i] = c;
                if (i == 0) mx = fmax(mx, c);
            }
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        flags |= __shfl_xor_sync(0xffffffffu, flags, o);
    }
    if (lane == 0) s_wmx[warp] = mx;
    if (lane == 0 && flags) atomicOr(&s_bad, flags);
    __syncthreads();
    if (s_bad) {   // nothing has been stored into another CTA yet
        if (rank == 0 && tid == 0) {
            const int f = s_bad;
            set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, (f & 2) ? 11 : ((f & 1) ? 10 : 15));
            if (a.do_permute) {
                a.hdr->n_active = 0;
                a.hdr->n_gtiles = 0;
                a.hdr->n_vgroups = 0;
            }
        }
        return;
    }
    mx = s_wmx[0];
    for (int w = 1; w < kClWarps; ++w) mx = fmax(mx, s_wmx[w]);
    const double budget = __dmul_rn(target, static_cast<double>(P));
    const int nb = static_cast<int>(floor(budget));
    double lo = 0.0;
    double hi = __dadd_rn(__dmul_rn(2.0, mx), 1.0);

    int round = 0;
    for (int it = 0; it < 64; ++round) {
        const int D = min(round < kClPruneRound ? kClDepthEarly : kClDepth, 64 - it);
        const int nn = (1 << D) - 1;
        const int par = round & 1, buf = round % 3;
        if (round == kClPruneRound) {   // the pairs whose choice no longer changes leave the list
            double klo[4], khi[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                klo[i] = __dmul_rn(lo, kv.v[i]);
                khi[i] = __dmul_rn(hi, kv.v[i]);
            }
            if (tid == 0) s_nl = 0;
            __syncthreads();
            int fixed = 0;
            for (int b = warp * 32; b < P; b += blockDim.x) {
                const int p = b + lane;
                bool keep = false;
                if (p < P) {
                    const double* c = s_c + p * nk;
                    double vlo[4], vhi[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        vlo[i] = i < nk ? __dadd_rn(c[i], klo[i]) : 0.0;
                        vhi[i] = i < nk ? __dadd_rn(c[i], khi[i]) : 0.0;
                    }
                    int ia = 0;
                    double va = vhi[0];
#pragma unroll
                    for (int i = 1; i < 4; ++i)
                        if (i < nk && vhi[i] < va) { va = vhi[i]; ia = i; }
                    bool same = true;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (i < nk && i != ia) same = same && (i < ia ? va < vlo[i] : va <= vlo[i]);
                    if (same) {
                        fixed += a.kmin + ia;
                        s_kf[p] = static_cast<uint8_t>(a.kmin + ia);
                    } else {
                        keep = true;
                    }
                }
                const unsigned m = __ballot_sync(0xffffffffu, keep);
                int base = 0;
                if (lane == 0 && m) base = atomicAdd(&s_nl, __popc(m));
                base = __shfl_sync(0xffffffffu, base, 0);
                if (keep) s_list[base + __popc(m & ((1u << lane) - 1u))] = p;
            }
            for (int o = 16; o > 0; o >>= 1) fixed += __shfl_xor_sync(0xffffffffu, fixed, o);
            if (lane == 0 && fixed) atomicAdd(&s_fixed, fixed);
            __syncthreads();
        }
        if (tid == 0) mbar_arrive_expect_tx(&cs.rbar[par], static_cast<uint32_t>(nn) * 4u);
        // this CTA's nodes (0-based ids rank, rank + kClCtas, ...), wpn warps each (a power of
        // two: all warps share the nodes of a small tree); each warp computes its node's midpoint
        // and counts planes over its share of the listed pairs
        const int nloc = nn > rank ? (nn - rank + kClCtas - 1) / kClCtas : 0;
        int wpn = kClWarps;
        while (wpn > 1 && wpn * nloc > kClWarps) wpn >>= 1;
        const int j = warp / wpn, sw = warp - j * wpn;
        const int node = rank + kClCtas * j + 1;   // heap index
        int n = 0;
        if (j < nloc) {
            const int depth = 31 - __clz(node);
            double l = lo, h = hi;
            for (int lev = depth - 1; lev >= 0; --lev) {
                const double m = midpoint(l, h);
                if ((node >> lev) & 1) l = m; else h = m;
            }
            const double mid = midpoint(l, h);
            const int nl = s_nl, step = 32 * wpn;
            int n0 = 0, n1 = 0;
            int q = 32 * sw + lane;
            for (; q + step < nl; q += 2 * step) {   // two independent pairs per iteration
                n0 += choose_k(s_c + s_list[q] * nk, nk, a.kmin, kv, mid);
                n1 += choose_k(s_c + s_list[q + step] * nk, nk, a.kmin, kv, mid);
            }
            if (q < nl) n0 += choose_k(s_c + s_list[q] * nk, nk, a.kmin, kv, mid);
            n = __reduce_add_sync(0xffffffffu, n0 + n1);
        }
        if (wpn > 1) {   // the warps of a node meet in shared memory
            if (tid < kClNodesPerCta) s_part[tid] = 0;
            __syncthreads();
            if (j < nloc && lane == 0) atomicAdd(&s_part[j], n);
            __syncthreads();
            n = s_part[j < nloc ? j : 0];
        }
        if (j < nloc && sw == 0 && lane < kClCtas)   // the node's predicate, to every CTA
            st_async_s32(mapa_shared(smem_u32(&cs.pw[buf][node]), static_cast<uint32_t>(lane)), s_fixed + n > nb ? 1 : 0,
                         mapa_shared(smem_u32(&cs.rbar[par]), static_cast<uint32_t>(lane)));
        {   // every node's predicate of this round is here (bounded)
            bool ok = true;
            if (tid == 0) {
                const uint32_t parity = (round >> 1) & 1;
                if (!mbar_try_wait_acq_cluster(&cs.rbar[par], parity)) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait_acq_cluster(&cs.rbar[par], parity)) {
                        if (globaltimer() - t0 > kWaitNs) {
                            set_error(a.hdr, DPA_ERR_DEVICE_TIMEOUT, 0x252);
                            ok = false;
                            break;
                        }
                    }
                }
            }
            if (!__syncthreads_and(ok ? 1 : 0)) return;
        }
        int nd = 1;   // the D steps
        for (int lev = 0; lev < D; ++lev) {
            const int pr = cs.pw[buf][nd];
            const double m = midpoint(lo, hi);
            lo = pr ? m : lo;
            hi = pr ? hi : m;
            nd = 2 * nd + pr;
        }
        it += D;
    }
    // Every CTA has received all the predicates stored into it, and stores nothing more: the
    // others may exit. CTA 0 writes the plane counts (listed pairs choose at the final hi) and
    // groups the pairs.
    if (rank != 0) return;
    {
        const int nl = s_nl;
        for (int q = tid; q < nl; q += blockDim.x) {
            const int p = s_list[q];
            s_kf[p] = static_cast<uint8_t>(choose_k(s_c + p * nk, nk, a.kmin, kv, hi));
        }
    }
    __syncthreads();
    for (int p = tid; p < P; p += blockDim.x) {
        a.k_out[p] = s_kf[p];
        s_k[p] = s_kf[p];
    }
    if (tid == 0 && a.lambda_out) *a.lambda_out = hi;
    if (!a.do_permute) return;
    __syncthreads();
    group_pairs(a, smem, Ls, P, nk, s_k, s_tmp, s_scan5);
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
    bool coop_ran = false;
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
        coop_ran = true;
    }
    if (!coop_ran && a.policy == DPA_ALLOC_LAGRANGE && P >= kClMinPairs && P <= kSpecMaxP) {
        // mid-size batches: the bisection over a cluster of SMs, then CTA 0 groups the pairs
        // the grouping's layout, then every pair's costs, the pair list and the final counts
        const size_t smem = allocate_smem_bytes(P, a.E, nk, a.vrec != nullptr) + static_cast<size_t>(P) * nk * 8 +
                            static_cast<size_t>(P) * 5;
        cudaError_t err = cudaFuncSetAttribute(allocate_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
        if (err != cudaSuccess) return err;
        if (kClCtas > 8) {
            err = cudaFuncSetAttribute(allocate_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (err != cudaSuccess) return err;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kClCtas);
        cfg.blockDim = dim3(kClThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kClCtas;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        void* cargs[] = {&b};
        return cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(allocate_cluster_kernel), cargs);
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
