// Post-routing plane allocation and token->expert grouping.
//
// DPA-MoE, Abstract: chunks are allocated at inference time from the live router gate
// scores. DuoRate, Abstract: a Lagrangian rate-distortion allocation solved by a bisection.
// MatMoE, review "Core Contribution": a binary search sets the precision split so that the
// average bit-width meets a target.
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

#include "common.cuh"
#include "kernels.h"

namespace dpa {
namespace {

constexpr int kAllocThreads = 1024;       // maximum block size
constexpr int kSmemCostDoubles = 8192;    // costs kept in shared memory up to this many
constexpr int kSmallP = 64;               // up to this many pairs one warp runs the bisection

__device__ __forceinline__ int choose_k(const double* c, int nk, int kmin, double lam) {
    double best = __dadd_rn(c[0], __dmul_rn(lam, static_cast<double>(kmin)));
    int kb = kmin;
    for (int i = 1; i < nk; ++i) {
        const double cost = __dadd_rn(c[i], __dmul_rn(lam, static_cast<double>(kmin + i)));
        if (cost < best) { best = cost; kb = kmin + i; }
    }
    return kb;
}

__device__ __forceinline__ double midpoint(double lo, double hi) { return __dmul_rn(0.5, __dadd_rn(lo, hi)); }

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

// Shared-memory carve-up: [costs (if they fit)] [counts E*nk] [seg E*nk+1] [sorted P] [k P]
struct AllocSmem {
    size_t costs, counts, seg, sorted, kk, total;
    bool costs_in_smem;
};

__host__ __device__ inline AllocSmem alloc_smem_layout(int P, int E, int nk) {
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
    L.total = (off + 15) & ~static_cast<size_t>(15);
    return L;
}

__global__ void __launch_bounds__(kAllocThreads) allocate_kernel(AllocArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_tmp[32];
    __shared__ double s_max[32];
    __shared__ int s_ok;
    __shared__ double s_lohi[2];
    __shared__ unsigned char s_pred[2][kAllocThreads];
    const int P = a.T * a.K;
    const int nk = a.kmax - a.kmin + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const AllocSmem Ls = alloc_smem_layout(P, a.E, nk);
    double* c_base = Ls.costs_in_smem ? reinterpret_cast<double*>(smem + Ls.costs) : a.cbuf;
    uint8_t* s_k = smem + Ls.kk;

    if (tid == 0) {
        const double tg = *a.target;
        s_ok = (tg >= static_cast<double>(a.kmin) && tg <= static_cast<double>(a.kmax)) ? 1 : 0;
        if (!s_ok) set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 10);
    }
    __syncthreads();
    int bad = 0;
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = a.idx[p];
        bad |= (e < 0 || e >= a.E) ? 1 : 0;
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0) { set_error(a.hdr, DPA_ERR_DEVICE_INVALID_INPUT, 11); s_ok = 0; }
    }
    __syncthreads();
    if (!s_ok) {
        if (a.do_permute && tid == 0) a.hdr->n_active = 0;
        return;
    }
    const double target = *a.target;

    // costs c[p][i] = fl(g_p * r_{e_p}(kmin + i))
    double mx = 0.0;
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = a.idx[p];
        const double g = a.gate[p];
        for (int i = 0; i < nk; ++i) {
            const double c = __dmul_rn(g, a.rtable[static_cast<size_t>(e) * a.B + (a.kmin + i - 1)]);
            c_base[static_cast<size_t>(p) * nk + i] = c;
            if (i == 0) mx = fmax(mx, c);
        }
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_max[warp] = mx;
    __syncthreads();
    mx = s_max[0];
    for (int w = 1; w < nw; ++w) mx = fmax(mx, s_max[w]);

    const double budget = __dmul_rn(target, static_cast<double>(P));
    double lo = 0.0;
    double hi = __dadd_rn(__dmul_rn(2.0, mx), 1.0);

    if (P <= kSmallP) {
        // one warp: lane n-1 evaluates node n of a depth-5 tree of midpoints, predicates come
        // back as a ballot and every lane walks the tree in registers (no block barriers)
        if (warp == 0) {
            for (int it = 0; it < 64;) {
                const int D = min(5, 64 - it);
                const int node = lane + 1;
                int pred = 0;
                if (node < (1 << D)) {
                    const int depth = 31 - __clz(node);
                    double l = lo, h = hi;
                    for (int lev = depth - 1; lev >= 0; --lev) {
                        const double m = midpoint(l, h);
                        if ((node >> lev) & 1) l = m; else h = m;
                    }
                    const double mid = midpoint(l, h);
                    int n = 0;
                    for (int p = 0; p < P; ++p) n += choose_k(c_base + p * nk, nk, a.kmin, mid);
                    pred = static_cast<double>(n) > budget ? 1 : 0;
                }
                const unsigned mask = __ballot_sync(0xffffffffu, pred);   // bit (node-1)
                int nd = 1;
                for (int lev = 0; lev < D; ++lev) {
                    const int pr = (mask >> (nd - 1)) & 1;
                    const double m = midpoint(lo, hi);
                    if (pr) lo = m; else hi = m;
                    nd = 2 * nd + pr;
                }
                it += D;
            }
            if (lane == 0) { s_lohi[0] = lo; s_lohi[1] = hi; }
        }
        __syncthreads();
        lo = s_lohi[0];
        hi = s_lohi[1];
    } else {
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
        for (int it = 0; it < 64; ++round) {
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
                for (int p = glane; p < P; p += gs) local += choose_k(c_base + static_cast<size_t>(p) * nk, nk, a.kmin, mid);
            }
            // every lane of the warp takes part in the group reduction (inactive lanes add 0)
            for (int o = gs >> 1; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
            if (active && glane == 0) s_pred[round & 1][node] = static_cast<double>(local) > budget ? 1 : 0;
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
        const int k = choose_k(c_base + static_cast<size_t>(p) * nk, nk, a.kmin, hi);
        a.k_out[p] = static_cast<uint8_t>(k);
        s_k[p] = static_cast<uint8_t>(k);
    }
    if (tid == 0 && a.lambda_out) *a.lambda_out = hi;
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
    for (int p = tid; p < P; p += blockDim.x) {
        const int key = a.idx[p] * nk + (s_k[p] - a.kmin);
        const int pos = atomicAdd(&s_counts[key], 1);
        s_sorted[pos] = p;
        a.pair_pos[p] = pos;
    }
    __syncthreads();
    // per-expert descriptors and two-token tiles (tiles never straddle k classes); experts in
    // rounds of blockDim so that the active list stays in ascending expert order
    int rank_base = 0, tile_base = 0;
    for (int e0 = 0; e0 < a.E; e0 += blockDim.x) {
        const int e = e0 + tid;
        int km = 0, ntiles = 0;
        if (e < a.E) {
            for (int i = 0; i < nk; ++i) {
                const int n = s_seg[e * nk + i + 1] - s_seg[e * nk + i];
                if (n > 0) km = a.kmin + i;
                ntiles += (n + 1) >> 1;
            }
        }
        const int flag = km > 0 ? 1 : 0;
        const int rank_incl = block_incl_scan(flag, s_tmp);
        const int tiles_incl = block_incl_scan(ntiles, s_tmp);
        const int rank = rank_base + rank_incl - flag;
        const int tile_off = tile_base + tiles_incl - ntiles;
        if (flag) {
            a.exp_desc[rank] = make_int4(e, km, ntiles, tile_off);
            int t = tile_off;
            for (int i = 0; i < nk; ++i) {
                const int s0 = s_seg[e * nk + i];
                const int n = s_seg[e * nk + i + 1] - s0;
                for (int j = 0; j < n; j += 2) {
                    const int posA = s0 + j, posB = j + 1 < n ? s0 + j + 1 : -1;
                    const int tokA = s_sorted[posA] / a.K;
                    const int tokB = posB >= 0 ? s_sorted[posB] / a.K : -1;
                    a.tiles[t++] = make_int4(a.kmin + i, posA, posB, (tokA & 0xFFFF) | ((tokB & 0xFFFF) << 16));
                }
            }
        }
        // totals of this round (the last thread's inclusive sums), broadcast
        if (tid == blockDim.x - 1) { s_tmp[0] = rank_incl; s_tmp[1] = tiles_incl; }
        __syncthreads();
        rank_base += s_tmp[0];
        tile_base += s_tmp[1];
        __syncthreads();
    }
    if (tid == 0) a.hdr->n_active = static_cast<uint32_t>(rank_base);
}

}  // namespace

size_t allocate_smem_bytes(int P, int E, int nk) { return alloc_smem_layout(P, E, nk).total; }

int allocate_threads(int P) { return P <= kSmallP ? 128 : kAllocThreads; }

cudaError_t launch_allocate(const AllocArgs& a, cudaStream_t stream) {
    const int nk = a.kmax - a.kmin + 1;
    const int P = a.T * a.K;
    const size_t smem = allocate_smem_bytes(P, a.E, nk);
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(allocate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
        if (err != cudaSuccess) return err;
    }
    allocate_kernel<<<1, allocate_threads(P), smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace dpa
