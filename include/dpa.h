/*
 * dpa.h - C ABI of the B200 (sm_100a) routed MoE expert FFN over prefix-decodable
 * bitplane weights.
 *
 * The method (pages cited by title and section):
 *  - DPA-MoE: A Runtime Precision Control Framework for MoE Inference, Abstract:
 *    expert weights in chunks that decode by prefix under one shared scale (the page's
 *    SharedScale AnyBCQ); each expert's reconstruction error measured ahead of time; the
 *    chunk count of each routed pair chosen after routing from the current gate scores,
 *    so one encoded layer serves many weight budgets.
 *  - DuoRate: Two-Rate Per-Expert Precision Allocation for MoE Serving, Abstract:
 *    one stored copy read by prefix, a precomputed distortion table, per-expert rates
 *    from a Lagrangian rate/distortion trade-off found by bisection; prefill reads every
 *    stored plane.
 *  - MatMoE: Matryoshka Mixture-of-Experts with Dynamic Mixed-Precision Quantization,
 *    Abstract and review section "Core Contribution": bitplane storage,
 *    floor-and-compensation (keep the top k of B code bits and add (2^(B-k)-1)/2),
 *    routing-score driven per-expert bit-widths under a target average bit-width.
 *
 * Conventions for every call:
 *  - Return value: DPA_OK or an error code; on error nothing has been launched and no
 *    output has been written.
 *  - "device" pointers are CUDA global memory owned by the caller; "host" pointers are
 *    ordinary CPU memory owned by the caller. The library never allocates, frees or
 *    keeps pointers between calls. Device calls are asynchronous on the given stream,
 *    never synchronise (except dpa_device_status) and copy nothing back to the host, so
 *    a sequence of them can be captured in a CUDA graph.
 *  - Every device buffer must be 16-byte aligned (bulk copies), else DPA_ERR_INVALID_ARG.
 *  - Errors found on the device (an out-of-range routed expert id passed to
 *    dpa_allocate, a bounded wait that ran out) set a flag in the workspace; read and
 *    clear it with dpa_device_status.
 *  - Matrices are row-major. Token activations and router weights are bf16 bit patterns.
 */
#ifndef DPA_H
#define DPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dpa_status {
    DPA_OK = 0,
    DPA_ERR_INVALID_ARG = 1,         /* bad pointer, size, alignment or descriptor field   */
    DPA_ERR_UNSUPPORTED = 2,         /* shape outside what the kernels handle (see below)  */
    DPA_ERR_WORKSPACE = 3,           /* workspace smaller than dpa_forward_workspace_size  */
    DPA_ERR_CUDA = 4,                /* a CUDA runtime call failed                          */
    DPA_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device wait ran out (reported by status) */
    DPA_ERR_DEVICE_INVALID_INPUT = 6 /* device data out of range (reported by status)      */
} dpa_status;

enum { DPA_FMT_UNIFORM = 0, DPA_FMT_BCQ = 1 };
enum { DPA_MAT_GATE = 0, DPA_MAT_UP = 1, DPA_MAT_DOWN = 2 };

/* One MoE layer. gate/up are [inter][hidden], down is [hidden][inter] per expert.
 *  format    DPA_FMT_UNIFORM: asymmetric B-bit codes, per-group fp16 scale s and zero z
 *                             shared by every k; the first k planes read with
 *                             floor-and-compensation: w = s*((q>>(B-k))*2^(B-k)
 *                             + (2^(B-k)-1)/2 - z).
 *            DPA_FMT_BCQ:     w = sum_{i<k} alpha_i * b_i, b_i in {-1,+1}, per-group fp16
 *                             alpha_i (binary-coded quantisation, greedy fit).
 *  bits      B, the stored planes (1..4).   kmin..kmax: planes a routed pair may read.
 *  group     G, inputs per scale group.     norm_topk: 1 = softmax over the top_k
 *            selected logits, 0 = softmax over all experts (then the top_k values).
 *  n_shared  always-on experts run densely in bf16 (not allocated, not in the budget).
 * Supported by the kernels: hidden, inter multiples of 64 and of group; group a multiple
 * of 64 and at most 512; bits <= 4; n_experts <= 1024; top_k <= 32; n_shared <= 8; a work
 * item's staging must fit in shared memory (else DPA_ERR_UNSUPPORTED). */
typedef struct dpa_layer_desc {
    int32_t hidden, inter, n_experts, top_k, n_shared;
    int32_t format, bits, kmin, kmax, group, norm_topk;
} dpa_layer_desc;

/* Bytes of one encoded layer (all routed experts).
 *  planes: bit planes. For expert e and matrix m (rows R, cols C), plane p (p = 0 is the
 *          most significant code bit, or the first BCQ sign plane) occupies R*C/8 bytes;
 *          the B planes of (e, m) are stored one after another, so the first k planes of a
 *          matrix are one contiguous prefix of its bytes. Matrices follow in the order
 *          gate, up, down; experts follow in order.
 *          Inside a plane the bits are in the decode kernel's fragment order: 16-row tiles,
 *          then 64-column blocks, then 32 lanes of one 32-bit word. Lane l = 4*g + c holds
 *          rows {g, g+8}; for rho in 0..3 and m in 0..7 the weight at
 *            row    = tile*16 + g + 8*(rho & 1)
 *            column = block*64 + 32*(m & 1) + 16*(rho >> 1) + 4*c + (m >> 1)
 *          sits at bit 4*m + rho of the word (DPA_FMT_BCQ), or at bit
 *          (4*m + (B-1-p) - rho) mod 32 in plane p (DPA_FMT_UNIFORM: rotated per plane, so
 *          that a decoder merges the planes under fixed masks and rotates once per rho).
 *          Use dpa_export_codes to read codes back in natural order.
 *  meta:   DPA_FMT_UNIFORM: per (e, m, row, group) an fp16 pair {s, z}, row-major,
 *          [E][3][R][C/G] with the three matrices in order.
 *          DPA_FMT_BCQ: per (e, m, plane, row, group) one fp16 alpha, [E][3][B][R][C/G]
 *          (the first k planes' alphas are a contiguous prefix per (e, m)).
 *  rtable: fp64 [E][B]; rtable[e][k-1] = ||W_e - W_e^(k)||_F^2 summed over gate, up, down.
 *  *_matrix_offset: byte offset of matrix m of expert e is
 *          e*planes_per_expert + planes_matrix_offset[m] (likewise for meta). */
typedef struct dpa_sizes {
    uint64_t planes_bytes, meta_bytes, rtable_bytes;
    uint64_t planes_per_expert, meta_per_expert;
    uint64_t planes_matrix_offset[3], meta_matrix_offset[3];
} dpa_sizes;

/* Device weights of one layer for dpa_moe_forward. planes/meta/rtable as written by
 * dpa_encode and copied to the device unchanged. w_router: bf16 [n_experts][hidden].
 * shared_*: bf16 dense always-on experts, gate/up [n_shared][inter][hidden],
 * down [n_shared][hidden][inter]; NULL when n_shared == 0. */
typedef struct dpa_layer_weights {
    const void* planes;
    const void* meta;
    const double* rtable;
    const void* w_router;
    const void* shared_gate;
    const void* shared_up;
    const void* shared_down;
    /* Per-expert stored widths (MatMoE, review "Core Contribution": each expert's maximum
     * bit-width, chosen offline under a memory budget). Both NULL: every expert holds all B
     * planes in the layout of dpa_encode. Both set: the layer is the compact blob of
     * dpa_compact_layer, expert_width uint8 [E] (device) holds each expert's stored planes
     * (kmin..kmax) and expert_offsets uint64 [E][2] (device) the byte offsets of each expert's
     * planes and scale data in `planes` and `meta`; every allocation policy then reads at most
     * expert_width[e] planes of expert e (the Lagrangian optimises within the widths; the other
     * policies' counts are clipped to them). The compact layout runs the decode GEMV kernels
     * only (DPA_PATH_TC returns DPA_ERR_UNSUPPORTED). */
    const uint8_t* expert_width;
    const uint64_t* expert_offsets;
} dpa_layer_weights;

/* Optional device outputs of dpa_moe_forward's decision path (any field may be NULL).
 * topk_idx int32 [T][top_k]; topk_gate fp64 [T][top_k]; k uint8 [T][top_k] (planes read
 * by each routed pair); lambda fp64 scalar (the final Lagrange multiplier);
 * pair_out fp32 [T][top_k][hidden]: each routed pair's expert output before the gate
 * weighting (diagnostic; costs T*top_k*hidden*4 bytes of writes).
 * events: optional cudaEvent_t handles (any may be NULL) recorded on the stream at the
 * stage boundaries of dpa_moe_forward: [0] before routing, [1] after routing, [2] after
 * allocation and grouping, [3] after the shared experts, [4] after the gate/up GEMV,
 * [5] after the down GEMV, [6] after the combine. Recording also works under stream
 * capture, so per-stage device times can be read from a replayed CUDA graph. On the
 * tensor-core path [4] and [5] follow the gate/up and down GEMMs.
 * expert_path: which kernels run the routed experts' FFN (same results up to the
 * rounding of fp32 accumulation and of the fp16 SwiGLU intermediate on the tensor-core path):
 *   DPA_PATH_AUTO (0)  tensor-core GEMMs when the format is uniform, hidden % 256 == 0,
 *                      inter % 256 == 0, the group is a power of two and the batch routes at
 *                      least DPA_TC_MIN_PAIRS_PER_EXPERT
 *                      pairs per expert on average (T*top_k >= that * n_experts); else GEMV;
 *   DPA_PATH_GEMV (1)  the batched GEMV kernels (any shape check_desc accepts);
 *   DPA_PATH_TC (2)    the tcgen05 grouped GEMMs (DPA_ERR_UNSUPPORTED when the shape does
 *                      not qualify as above, minus the pairs-per-expert condition). */
#define DPA_PATH_AUTO 0
#define DPA_PATH_GEMV 1
#define DPA_PATH_TC 2
#define DPA_TC_MIN_PAIRS_PER_EXPERT 16
/* alloc_policy: how the routed pairs' plane counts are chosen (see dpa_allocate_ex); threshold:
 * device fp64 scalar read by DPA_ALLOC_THRESHOLD (NULL otherwise); expert_k: device uint8 [E]
 * read by DPA_ALLOC_EXPERT_TABLE (NULL otherwise). With alloc_policy = 0 the Lagrangian
 * allocation of dpa_allocate runs. */
typedef struct dpa_aux {
    int32_t* topk_idx;
    double* topk_gate;
    uint8_t* k;
    double* lambda;
    float* pair_out;
    void* events[7];
    int32_t expert_path;
    int32_t alloc_policy;
    const double* threshold;
    const uint8_t* expert_k;
} dpa_aux;

/* Validate a descriptor and return the encoded sizes. Host only. */
dpa_status dpa_encoded_sizes(const dpa_layer_desc* desc, dpa_sizes* out);

/* Offline encoder (host, synchronous, multithreaded with n_threads >= 1 or 0 = all cores).
 * Encodes routed experts [e_begin, e_begin + n_e) of the layer.
 * w_gate, w_up: host fp32 [n_e][inter][hidden]; w_down: host fp32 [n_e][hidden][inter]
 * (the experts to encode, contiguous). planes, meta, rtable: host buffers sized for the
 * WHOLE layer (dpa_encoded_sizes); only the parts of experts e_begin.. are written.
 * Uniform codes per group of G inputs (DPA-MoE "SharedScale"; MatMoE shared quantisation
 * parameters): lo/hi = group min/max, s = fp16((hi-lo)/(2^B-1)) (1 if it rounds to 0),
 * z = clamp(rint(-lo/s), 0, 2^B-1), q = clamp(rint(w/s)+z, 0, 2^B-1), rint ties to even,
 * fp64 arithmetic. BCQ per group: for each plane i, b_i = sign(R) (sign(0) = +1),
 * alpha_i = fp16(sum|R|/G) (sequential sum), R -= alpha_i*b_i. rtable[e][k-1] is a
 * sequential fp64 sum of (w - w_k)^2 over gate, up, down in row-major order.
 * Errors: DPA_ERR_INVALID_ARG for NULL pointers, a range outside [0, n_experts), or a
 * group whose scale does not fit fp16. */
dpa_status dpa_encode(const dpa_layer_desc* desc, int e_begin, int n_e,
                      const float* w_gate, const float* w_up, const float* w_down,
                      void* planes, void* meta, double* rtable, int n_threads);

/* Read codes of one encoded matrix back in natural order (host). codes: uint8 [R][C];
 * code = sum_p plane_p << (B-1-p) over all B planes. */
dpa_status dpa_export_codes(const dpa_layer_desc* desc, const void* planes, int expert,
                            int matrix, uint8_t* codes);

/* Read one matrix's scale data back as fp32 (host). Uniform: s_or_alpha [R][C/G] = s,
 * zero [R][C/G] = z. BCQ: s_or_alpha [B][R][C/G] = alpha, zero unused (may be NULL). */
dpa_status dpa_export_meta(const dpa_layer_desc* desc, const void* meta, int expert,
                           int matrix, float* s_or_alpha, float* zero);

/* Router (device). Defined by: DPA-MoE: A Runtime Precision Control Framework for MoE
 * Inference, Abstract (each token is sent to a small set of experts by the router, and
 * the live gate scores then drive the allocation); the softmax/top-k gating form is the
 * plainest reading, the pages print no formula for it.
 * Logits l[t][e] = the exact dot product of bf16 x[t] and bf16
 * w_router[e], rounded once to fp64; top_k experts by descending logit (ties to the lower
 * id); gates as described at dpa_layer_desc.norm_topk, using a fixed fp64 exp (Cody-Waite
 * reduction with ln 2 in two parts, degree-13 Taylor polynomial, results below 2^-1021
 * flushed to 0). Decisions are bit-identical to any IEEE implementation of the same steps.
 * x: device bf16 [n_tokens][hidden]; w_router: device bf16 [n_experts][hidden];
 * topk_idx: device int32 [n_tokens][top_k]; topk_gate: device fp64 [n_tokens][top_k];
 * logits: optional device fp64 [n_tokens][n_experts] (NULL to skip).
 * ws: device workspace of dpa_forward_workspace_size(desc, n_tokens) bytes. */
dpa_status dpa_route(const dpa_layer_desc* desc, const void* x, int n_tokens,
                     const void* w_router, int32_t* topk_idx, double* topk_gate,
                     double* logits, void* ws, size_t ws_bytes, void* stream);

/* Plane allocation (device). For the P = n_tokens*top_k routed pairs (token-major, slot
 * order) with expert e and gate g, and a multiplier lambda, each pair reads
 *     k(lambda) = argmin_{kmin<=k<=kmax} fl(fl(g*rtable[e][k-1]) + fl(lambda*k))
 * planes (ties to the smaller k). lambda comes from exactly 64 fp64 bisection steps on
 * [0, 2*max_p fl(g_p*rtable[e_p][kmin-1]) + 1]: mid = 0.5*(lo+hi); if sum_p k_p(mid) >
 * target*P then lo = mid else hi = mid; the result is lambda = hi and k = k(hi), so the
 * mean planes per pair never exceeds the target (DuoRate Lagrangian bisection; MatMoE
 * binary search to a target average bit-width).
 * target_bpw: device fp64 scalar in [kmin, kmax] (a device value so one captured graph
 * serves every budget; out of range -> k and lambda untouched, device flag
 * DPA_ERR_DEVICE_INVALID_INPUT). k_out: device uint8 [n_tokens][top_k];
 * lambda_out: device fp64 scalar (may be NULL). */
dpa_status dpa_allocate(const dpa_layer_desc* desc, const double* rtable,
                        const int32_t* topk_idx, const double* topk_gate, int n_tokens,
                        const double* target_bpw, uint8_t* k_out, double* lambda_out,
                        void* ws, size_t ws_bytes, void* stream);

/* Allocation policies (dpa_allocate_ex, dpa_aux.alloc_policy):
 *  DPA_ALLOC_LAGRANGE (0)  the gate-driven Lagrangian allocation of dpa_allocate (DPA-MoE,
 *                          Abstract; DuoRate, Abstract). lambda_out = the final multiplier.
 *  DPA_ALLOC_UNIFORM (1)   the control DPA-MoE, Abstract, compares with: uniform chunk
 *                          allocation at a matched budget. The budget floor(target*P) planes
 *                          is shared equally: every pair reads floor(budget/P) planes and the
 *                          first (budget mod P) pairs in token-major slot order one more; the
 *                          gates are ignored. lambda_out = 0.
 *  DPA_ALLOC_THRESHOLD (2) MatMoE, review "Core Contribution": a pair whose routing score (its
 *                          gate) is above a threshold reads kmax planes, every other pair kmin.
 *                          The threshold comes from dpa_calibrate_threshold ahead of time; no
 *                          budget is enforced on the live batch. target_bpw is not read (may be
 *                          NULL). lambda_out = the threshold.
 *  DPA_ALLOC_EXPERT_TABLE (3) DuoRate, Abstract: every pair routed to expert e reads expert_k[e]
 *                          planes, a per-workload table solved ahead of time by
 *                          dpa_solve_expert_rates. target_bpw is not read (may be NULL).
 *                          lambda_out = 0. */
#define DPA_ALLOC_LAGRANGE 0
#define DPA_ALLOC_UNIFORM 1
#define DPA_ALLOC_THRESHOLD 2
#define DPA_ALLOC_EXPERT_TABLE 3

/* dpa_allocate with a choice of policy (device). Arguments as dpa_allocate, plus
 * policy (above); threshold: device fp64 scalar, read by DPA_ALLOC_THRESHOLD only (a NaN or
 * infinite threshold sets the device flag DPA_ERR_DEVICE_INVALID_INPUT and leaves k untouched);
 * expert_k: device uint8 [n_experts], read by DPA_ALLOC_EXPERT_TABLE only (an entry outside
 * [kmin, kmax] for a routed expert sets the same flag). rtable is read by DPA_ALLOC_LAGRANGE only.
 * Errors: DPA_ERR_INVALID_ARG for an unknown policy or a missing input of the policy. */
dpa_status dpa_allocate_ex(const dpa_layer_desc* desc, int policy, const double* rtable,
                           const int32_t* topk_idx, const double* topk_gate, int n_tokens,
                           const double* target_bpw, const double* threshold, const uint8_t* expert_k,
                           uint8_t* k_out, double* lambda_out, void* ws, size_t ws_bytes, void* stream);

/* Distortion tensor of the workload-profiled read rates (host, synchronous). Defined by:
 * DuoRate, Abstract (a distortion tensor baked offline beside the stored weights). For routed
 * experts [e_begin, e_begin + n_e): T[e][k-1][j] = sum over the rows of gate, then of up, of
 * (w - w_k)^2 at input channel j, w_k the stored code read at k planes (one sequential fp64 sum
 * per channel, rows in order). w_gate, w_up: host fp32 [n_e][inter][hidden] (the experts'
 * original weights); planes, meta: the host output of dpa_encode for the whole layer;
 * T: host fp64 [n_experts][bits][hidden] (only the given experts' parts are written).
 * n_threads >= 1, or 0 for all cores. */
dpa_status dpa_distortion_tensor(const dpa_layer_desc* desc, int e_begin, int n_e, const float* w_gate,
                                 const float* w_up, const void* planes, const void* meta, double* T,
                                 int n_threads);

/* Workload profile of a prefill (device). Defined by: DuoRate, Abstract (the workload's own
 * prefill is profiled, without labels). m[j] = (sum over tokens in order of x[t][j]^2) / T in
 * fp64; counts[e] = pairs of topk_idx routed to e. x: device bf16 [n_tokens][hidden];
 * topk_idx: device int32 [n_tokens][top_k] (dpa_route's output); m: device fp64 [hidden];
 * counts: device int32 [n_experts] (overwritten). An out-of-range expert id sets the device
 * flag DPA_ERR_DEVICE_INVALID_INPUT. ws: at least dpa_forward_workspace_size(desc, 1) bytes. */
dpa_status dpa_profile_prefill(const dpa_layer_desc* desc, const void* x, int n_tokens,
                               const int32_t* topk_idx, double* m, int32_t* counts, void* ws,
                               size_t ws_bytes, void* stream);

/* Per-expert decode read rates from a workload profile (device). Defined by: DuoRate, Abstract
 * (a Lagrangian rate/distortion allocation under the decode functional, one dot product per
 * expert and a bisection; routing frequency cancels from each expert's decision).
 * D_e(k) = <m, T[e][k-1]> summed as 32 chunks of hidden/32 channels (each sequential) combined
 * by the pairwise tree p[i]+p[i+16], +[i+8], +[i+4], +[i+2], +[i+1];
 * k_e(lambda) = argmin_{kmin<=k<=kmax} fl(D_e(k) + fl(lambda*k)), ties to the smaller k;
 * 64 fp64 bisection steps on [0, 2 max_e D_e(kmin) + 1]: if sum_e counts[e]*k_e(mid) >
 * target*sum_e counts[e] then lo = mid else hi = mid; k_table[e] = k_e(hi) for every expert.
 * T: device fp64 [n_experts][bits][hidden]; m, counts as from dpa_profile_prefill;
 * target_bpw: device fp64 scalar in [kmin, kmax] (else the device flag
 * DPA_ERR_DEVICE_INVALID_INPUT, table untouched); k_table: device uint8 [n_experts];
 * lambda_out: device fp64 scalar or NULL. ws: at least dpa_forward_workspace_size(desc, 1). */
dpa_status dpa_solve_expert_rates(const dpa_layer_desc* desc, const double* T, const double* m,
                                  const int32_t* counts, const double* target_bpw, uint8_t* k_table,
                                  double* lambda_out, void* ws, size_t ws_bytes, void* stream);

/* Threshold of DPA_ALLOC_THRESHOLD from a calibration set of routing scores (device).
 * Defined by: MatMoE, review "Core Contribution" (a binary search over a calibration score
 * distribution sets the threshold so that the average bit-width meets the target).
 * scores: device fp64 [n_scores], the gates of a calibration batch's routed pairs (for
 * example dpa_route's topk_gate on calibration tokens). 64 fp64 bisection steps on [0, 1]:
 *   mid = 0.5*(lo+hi); planes = kmin*n + (kmax-kmin)*#{s > mid};
 *   if planes > target*n then lo = mid else hi = mid;
 * threshold_out (device fp64 scalar) = hi, so the calibration set's average plane count is at
 * most the target. target_bpw: device fp64 scalar in [kmin, kmax] (else the device flag
 * DPA_ERR_DEVICE_INVALID_INPUT, threshold untouched). ws: at least
 * dpa_forward_workspace_size(desc, 1) bytes (its error flag is used). */
dpa_status dpa_calibrate_threshold(const dpa_layer_desc* desc, const double* scores, int n_scores,
                                   const double* target_bpw, double* threshold_out, void* ws,
                                   size_t ws_bytes, void* stream);

/* Allocation-free variant of dpa_route, for callers that cannot allocate device memory:
 * for example a plugin whose host engine owns every byte of device memory, or a loop that
 * must not call the allocator. It has no counterpart in the pages; it exists for those callers.
 * Same inputs, outputs and decisions as dpa_route, but no workspace: its scratch (per-token
 * counters and a logits buffer) lives in a fixed array of about 0.5 MB inside the library,
 * which every GPU that loads the library holds until the process exits.
 * Limits: n_tokens <= 1024 and n_tokens * n_experts <= 65536, else DPA_ERR_UNSUPPORTED
 * (nothing launched). Every batch runs the router's per-logit kernel (dpa_route switches to
 * its tiled kernels from 2 tokens; the decisions are the same). The first call on a device
 * looks up the array's device address, so make it before any stream capture; the address is
 * kept for the life of the process, so resetting the device (cudaDeviceReset) after that first
 * call is not supported. Every call shares the array: calls whose executions
 * overlap on the GPU (other streams, other threads) race and must be serialised by the
 * caller. Device-side input checks (NaN/Inf tokens) are not reported by this variant.
 * logits may be NULL. stream: cudaStream_t. */
dpa_status dpa_route_noalloc(const dpa_layer_desc* desc, const void* x, int n_tokens,
                             const void* w_router, int32_t* topk_idx, double* topk_gate,
                             double* logits, void* stream);

/* Workspace bytes that dpa_route, dpa_allocate and dpa_moe_forward need for up to
 * max_tokens tokens. Returns 0 for an invalid descriptor. */
size_t dpa_forward_workspace_size(const dpa_layer_desc* desc, int max_tokens);

/* One MoE layer forward (device). Defined by: DPA-MoE: A Runtime Precision Control
 * Framework for MoE Inference, Abstract (post-routing allocation of prefix-decodable
 * chunks from live gate scores, one encoded layer at many budgets); MatMoE: Matryoshka
 * Mixture-of-Experts with Dynamic Mixed-Precision Quantization, review section "Core
 * Contribution" (bitplane storage read by prefix, floor-and-compensation); DuoRate:
 * Two-Rate Per-Expert Precision Allocation for MoE Serving, Abstract (the Lagrangian
 * bisection; a decode step pays only for the planes of the experts it selects).
 * Steps: route, allocate, group pairs by expert and plane
 * count, run each routed pair's SwiGLU expert reading only its first k planes
 *   a = W_gate^(k) x, u = W_up^(k) x, h = silu(a) * u, o = W_down^(k) h,
 * and write y[t] = bf16( sum_{slots} g * o  (+ dense shared experts) ).
 * x: device bf16 [n_tokens][hidden]; y: device bf16 [n_tokens][hidden];
 * target_bpw: device fp64 scalar (see dpa_allocate); aux: optional (may be NULL).
 * ws must hold dpa_forward_workspace_size(desc, n_tokens) bytes and is clobbered. */
dpa_status dpa_moe_forward(const dpa_layer_desc* desc, const dpa_layer_weights* weights,
                           const void* x, int n_tokens, const double* target_bpw, void* y,
                           dpa_aux* aux, void* ws, size_t ws_bytes, void* stream);

/* Glue between the layers of a stack of MoE layers (pre-norm residual):
 *   h += y                     (skipped when y is NULL)
 *   x  = bf16( h / sqrt(mean_j h_j^2 + 1e-6) )
 * h: device fp32 [n_tokens][hidden], the residual stream (updated in place);
 * y: device bf16 [n_tokens][hidden] (the previous layer's output) or NULL;
 * x: device bf16 [n_tokens][hidden], the next layer's input. hidden must be a multiple of 4.
 * The pages give no form for the glue; this is the plainest reading of a residual add and an
 * RMSNorm (unit weight) between the layers. */
dpa_status dpa_residual_rmsnorm(const void* y, float* h, int n_tokens, int hidden, void* x, void* stream);

/* Prefix streaming of offloaded experts (host -> device). Defined by: MatMoE, review section on
 * the SSD-offloading regime (nested bitplanes let an offloaded expert's low-precision prefix be
 * fetched on its own); DuoRate, Abstract (a weight stream readable by prefix).
 * For each listed expert experts[i] (host int32 [n]) copies the first kplanes[i] (host uint8 [n],
 * 1..bits) planes of its gate, up and down matrices from host_planes to the same offsets of
 * dev_planes - one contiguous prefix per matrix, one cudaMemcpyAsync each - and the scale data
 * those planes need from host_meta to dev_meta (uniform: the expert's scales and zeros;
 * binary-coded: the first kplanes[i] alpha planes of each matrix). host_* are encoded layers
 * (dpa_encode's layout), ideally page-locked so that the copies are asynchronous; dev_* are
 * device buffers of the same sizes. The bytes issued are written to *bytes_out (may be NULL).
 * After the copies complete, a forward whose pairs read at most kplanes[i] planes of expert
 * experts[i] reads only streamed bytes. Errors: DPA_ERR_INVALID_ARG for NULL pointers or an
 * expert id or plane count out of range (nothing issued). */
dpa_status dpa_stream_prefixes(const dpa_layer_desc* desc, const void* host_planes, const void* host_meta,
                               const int32_t* experts, const uint8_t* kplanes, int n, void* dev_planes,
                               void* dev_meta, uint64_t* bytes_out, void* stream);

/* ---- Per-expert stored widths ----
 * MatMoE, review "Core Contribution": offline, an ILP picks each expert's maximum bit-width
 * (2/3/4) under a memory budget, with the metric routing score x Fisher-approximated Hessian
 * x quantization error. Here the ILP is
 *     minimise sum_e fl(importance[e] * rtable[e][b_e - 1])
 *     subject to sum_e b_e <= budget_planes,  kmin <= b_e <= kmax,
 * solved exactly by dynamic programming over the experts from the last
 * (f(e, u) = min_b fl(fl(importance[e] rtable[e][b-1]) + f(e+1, u-b)), ties to the smaller b;
 * the widths are read off from u = min(budget, E kmax) forwards). Every plane of every expert
 * has the same size, so the memory budget is a count of stored planes over all experts.
 * importance: fp64 [E] (host), e.g. each expert's routing mass over a calibration batch (the sum
 * of its routed pairs' gates); no Fisher information is used (factor 1). rtable: fp64 [E][B]
 * (host, from dpa_encode). widths: uint8 [E] (host, written). Host, synchronous.
 * Errors: DPA_ERR_INVALID_ARG for NULL pointers, non-finite or negative importance, or a budget
 * below E * kmin. */
dpa_status dpa_solve_stored_widths(const dpa_layer_desc* desc, const double* importance, const double* rtable,
                                   int64_t budget_planes, uint8_t* widths);

/* Bytes of the compact layer for per-expert widths (host): expert e holds, per matrix (gate,
 * up, down in order), its first widths[e] planes (the prefix of dpa_encode's planes), then its
 * scale data (uniform: as in dpa_encode; binary-coded: the first widths[e] planes' alphas per
 * matrix). Errors: DPA_ERR_INVALID_ARG for NULL pointers or a width outside [kmin, kmax]. */
dpa_status dpa_compact_sizes(const dpa_layer_desc* desc, const uint8_t* widths, uint64_t* planes_bytes,
                             uint64_t* meta_bytes);

/* Builds the compact layer from dpa_encode's planes and meta (host buffers; planes_out and
 * meta_out of dpa_compact_sizes' sizes, caller-owned) and the per-expert byte offsets
 * offsets[e][0] (planes) and offsets[e][1] (meta), uint64 [E][2]. Experts follow in order.
 * Host, synchronous. Errors: as dpa_compact_sizes. */
dpa_status dpa_compact_layer(const dpa_layer_desc* desc, const void* planes, const void* meta, const uint8_t* widths,
                             void* planes_out, void* meta_out, uint64_t* offsets);

/* Test support for the device-side failure handling (the pages have no counterpart).
 * Runs one of the library's bounded device waits against a barrier that nothing completes,
 * with a limit of limit_ns (1e3 .. 2e9 ns) instead of the kernels' 200 ms:
 *   kind 0  the mbarrier wait of the bulk-copy and tensor-core pipelines;
 *   kind 1  the abortable wait of the expert GEMV (one warp times out, the others leave on the
 *           CTA's abort flag);
 *   kind 2  the grid barrier of the cooperative allocation, one of two CTAs held back.
 * The kernel returns after the limit and records DPA_ERR_DEVICE_TIMEOUT in ws's device flag
 * (read it with dpa_device_status); nothing else is written except, for kind 2, a counter at
 * byte 256 of ws. ws: device, 16-byte aligned, at least 512 bytes. */
dpa_status dpa_debug_timeout_probe(void* ws, size_t ws_bytes, int kind, uint64_t limit_ns, void* stream);

/* Synchronise `stream`, read the device error flag in ws, clear it, and return it
 * (DPA_OK if no device error was recorded). */
dpa_status dpa_device_status(void* ws, void* stream);

/* Human-readable name of a status code (static string). */
const char* dpa_status_string(dpa_status s);

/* Library version (major*10000 + minor*100 + patch). */
int dpa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DPA_H */
