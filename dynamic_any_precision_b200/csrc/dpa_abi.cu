// C ABI of the library (include/dpa.h): validation, sizes, workspace layout, launches.
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "common.cuh"
#include "dpa.h"
#include "kernels.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dpa_status check_desc(const dpa_layer_desc* d) {
    if (!d) return DPA_ERR_INVALID_ARG;
    if (d->hidden <= 0 || d->inter <= 0 || d->n_experts <= 0 || d->top_k <= 0 || d->group <= 0)
        return DPA_ERR_INVALID_ARG;
    if (d->format != DPA_FMT_UNIFORM && d->format != DPA_FMT_BCQ) return DPA_ERR_INVALID_ARG;
    if (d->bits < 1 || d->kmin < 1 || d->kmin > d->kmax || d->kmax > d->bits) return DPA_ERR_INVALID_ARG;
    if (d->norm_topk != 0 && d->norm_topk != 1) return DPA_ERR_INVALID_ARG;
    if (d->n_shared < 0 || d->top_k > d->n_experts) return DPA_ERR_INVALID_ARG;
    if (d->bits > 4 || d->n_experts > 1024 || d->top_k > 32 || d->n_shared > 8) return DPA_ERR_UNSUPPORTED;
    if (d->hidden % 64 || d->inter % 64 || d->group % 64 || d->group > 512) return DPA_ERR_UNSUPPORTED;
    if (d->hidden % d->group || d->inter % d->group) return DPA_ERR_UNSUPPORTED;
    if (d->hidden > 16384 || d->inter > 16384) return DPA_ERR_UNSUPPORTED;
    // the staging of the expert GEMV's small-batch variant must fit in shared memory
    if (dpa::vp_smem_bytes(d->hidden, d->group, d->format, d->bits, 2, 1) > dpa::kVpMaxSmem ||
        dpa::vp_smem_bytes(d->inter, d->group, d->format, d->bits, 1, 1) > dpa::kVpMaxSmem)
        return DPA_ERR_UNSUPPORTED;
    return DPA_OK;
}

// ---- workspace layout ----
struct WsLayout {
    size_t hdr, counters, logits, idx, gate, k, lambda, cbuf, pairpos, xdig, xscl, xfsx, h, out_pair, sh_h, sh_out,
        gtiles, postok, coop, rstats, rpart, vstart, xperm, hdig, hscl, hfsx, vrec, total;
};

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

constexpr int kVpMaxGrid = 512;   // CTAs of an expert GEMV launch the balanced start tables cover

WsLayout ws_layout(const dpa_layer_desc* d, int T) {
    WsLayout L;
    const size_t P = static_cast<size_t>(T) * d->top_k;
    const int nk = d->kmax - d->kmin + 1;
    const size_t E = d->n_experts, H = d->hidden, I = d->inter;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    L.hdr = take(sizeof(dpa::WsHeader));
    L.counters = take(sizeof(unsigned) * T);
    L.logits = take(8 * static_cast<size_t>(T) * E);
    L.idx = take(4 * P);
    L.gate = take(8 * P);
    L.k = take(P);
    L.lambda = take(8);
    L.cbuf = take(8 * P * nk);
    L.pairpos = take(4 * P);
    const size_t ngp_h = ((H / d->group) + 3) & ~static_cast<size_t>(3);
    const size_t ngp_i = ((I / d->group) + 3) & ~static_cast<size_t>(3);
    L.xdig = take(2 * static_cast<size_t>(T) * H);
    L.xscl = take(4 * static_cast<size_t>(T) * ngp_h);
    L.xfsx = take(4 * static_cast<size_t>(T) * ngp_h);
    L.h = take(4 * P * I);
    L.out_pair = take(4 * P * H);
    L.sh_h = take(4 * static_cast<size_t>(T) * d->n_shared * I);
    L.sh_out = take(4 * static_cast<size_t>(T) * H);
    L.gtiles = take(16 * (P / dpa::kGemmTileTokens + E * nk + 1));
    L.postok = take(4 * P);
    L.coop = take(sizeof(dpa::CoopSync));
    L.rstats = take((8 + 4 * (H / 64 + 1)) * (static_cast<size_t>(T) + E) + 32);
    L.rpart = take(8 * dpa::route_partial_doubles(T, static_cast<int>(E), static_cast<int>(H)));
    L.vstart = take(4 * 2 * (kVpMaxGrid + 1));
    L.xperm = take(2 * P * H);
    L.hdig = take(2 * P * I);
    L.hscl = take(4 * P * ngp_i);
    L.hfsx = take(4 * P * ngp_i);
    L.vrec = take(4 * dpa::kVRecInts * (P / 4 + E * nk + 1));
    L.total = off;
    return L;
}

int num_sms_current() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && cache[dev]) return cache[dev];
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (dev < 64) cache[dev] = n;
    return n;
}

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

}  // namespace

// Stage events of dpa_moe_forward: under stream capture they must be external event-record
// nodes so that the replayed graph records them.
struct StageMarks {
    const dpa_aux* aux;
    cudaStream_t s;
    cudaStreamCaptureStatus cap;
    void operator()(int i) const {
        if (!aux || !aux->events[i]) return;
        cudaEvent_t ev = static_cast<cudaEvent_t>(aux->events[i]);
        if (cap == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
        else cudaEventRecord(ev, s);
    }
};

// 5. combine: y[t] = bf16(sum over slots in order of gate * expert output (+ shared experts))
static dpa_status combine_stage(const dpa_layer_desc* d, const dpa_layer_weights* w, const double* gate, int T,
                                const dpa_aux* aux, void* y, void* ws, const WsLayout& L, dpa::WsHeader* hdr,
                                cudaStream_t s, const StageMarks& mark) {
    (void)w;
    const int K = d->top_k;
    dpa::CombineArgs ca{};
    ca.out_pair = at<float>(ws, L.out_pair);
    ca.pair_pos = at<int32_t>(ws, L.pairpos);
    ca.gate = gate;
    ca.shared_out = d->n_shared > 0 ? at<float>(ws, L.sh_out) : nullptr;
    ca.pair_out_user = aux ? aux->pair_out : nullptr;
    ca.y = static_cast<uint16_t*>(y);
    ca.T = T;
    ca.K = K;
    ca.H = d->hidden;
    ca.hdr = hdr;
    if (dpa::launch_combine(ca, s) != cudaSuccess) return DPA_ERR_CUDA;
    mark(6);
    return DPA_OK;
}

// Arguments of one expert GEMV launch of the forward: gate/up (down = false: x digits by token
// -> h [P][I]) or down (h digits by grouped position -> per-pair outputs [P][H]).
static dpa::VpArgs vp_launch_args(const dpa_layer_desc* d, const dpa_layer_weights* w, const dpa_sizes& sz, void* ws,
                                  const WsLayout& L, int T, int tpg, bool down) {
    dpa::VpArgs va{};
    const int P = T * d->top_k;
    const int nk = d->kmax - d->kmin + 1;
    va.planes = static_cast<const uint8_t*>(w->planes);
    va.meta = static_cast<const uint8_t*>(w->meta);
    va.planes_per_expert = sz.planes_per_expert;
    va.meta_per_expert = sz.meta_per_expert;
    for (int m = 0; m < 3; ++m) {
        va.planes_mat_off[m] = sz.planes_matrix_offset[m];
        va.meta_mat_off[m] = sz.meta_matrix_offset[m];
    }
    va.fmt = d->format;
    va.B = d->bits;
    va.G = d->group;
    va.tiles_per_group = tpg;
    va.vrec = at<int32_t>(ws, L.vrec);
    va.hdr = at<dpa::WsHeader>(ws, L.hdr);
    va.expert_off = w->expert_offsets;
    va.expert_width = w->expert_width;
    const int tiles_bound = P / 4 + d->n_experts * nk;
    va.max_groups = P < tiles_bound ? P : tiles_bound;
    if (!down) {
        va.R = d->inter;
        va.K = d->hidden;
        va.mat0 = 0;
        va.nmat = 2;
        va.dig = at<int8_t>(ws, L.xdig);
        va.dscl = at<float>(ws, L.xscl);
        va.dfsx = at<float>(ws, L.xfsx);
        va.dig_by_token = 1;
        va.out = at<float>(ws, L.h);
    } else {
        va.R = d->hidden;
        va.K = d->inter;
        va.mat0 = 2;
        va.nmat = 1;
        va.dig = at<int8_t>(ws, L.hdig);
        va.dscl = at<float>(ws, L.hscl);
        va.dfsx = at<float>(ws, L.hfsx);
        va.dig_by_token = 0;
        va.out = at<float>(ws, L.out_pair);
    }
    return va;
}

// Per-row exactness statistics of the large-batch router, carved from the workspace.
static void set_route_stats(dpa::RouteArgs& r, void* ws, const WsLayout& L, int T, int E) {
    unsigned char* base = at<unsigned char>(ws, L.rstats);
    r.n2_x = reinterpret_cast<double*>(base);
    r.n2_w = r.n2_x + T;
    const size_t lsb_off = (8 * (static_cast<size_t>(T) + E) + 15) & ~static_cast<size_t>(15);
    const size_t nrow = static_cast<size_t>(r.H / 64);   // H % 512 == 0 on the tiled path: 16-byte rows
    r.lsb_x = reinterpret_cast<int16_t*>(base + lsb_off);
    r.lsb_w = r.lsb_x + static_cast<size_t>(T) * nrow;
    r.hb_x = r.lsb_w + static_cast<size_t>(E) * nrow;
    r.hb_w = r.hb_x + static_cast<size_t>(T) * nrow;
    r.part = at<double>(ws, L.rpart);
}

extern "C" {

int dpa_version(void) { return 100; }

const char* dpa_status_string(dpa_status s) {
    switch (s) {
        case DPA_OK: return "ok";
        case DPA_ERR_INVALID_ARG: return "invalid argument";
        case DPA_ERR_UNSUPPORTED: return "unsupported shape";
        case DPA_ERR_WORKSPACE: return "workspace too small";
        case DPA_ERR_CUDA: return "CUDA error";
        case DPA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case DPA_ERR_DEVICE_INVALID_INPUT: return "invalid device input";
    }
    return "unknown status";
}

dpa_status dpa_encoded_sizes(const dpa_layer_desc* d, dpa_sizes* out) {
    const dpa_status st = check_desc(d);
    if (st != DPA_OK) return st;
    if (!out) return DPA_ERR_INVALID_ARG;
    const uint64_t H = d->hidden, I = d->inter, B = d->bits, G = d->group;
    const uint64_t mat_planes = B * H * I / 8;     // one matrix, all planes
    std::memset(out, 0, sizeof(*out));
    out->planes_matrix_offset[0] = 0;
    out->planes_matrix_offset[1] = mat_planes;
    out->planes_matrix_offset[2] = 2 * mat_planes;
    out->planes_per_expert = 3 * mat_planes;
    uint64_t mg, md;   // meta bytes of gate (= up) and down
    if (d->format == DPA_FMT_UNIFORM) {
        mg = I * (H / G) * 4;
        md = H * (I / G) * 4;
    } else {
        mg = B * I * (H / G) * 2;
        md = B * H * (I / G) * 2;
    }
    out->meta_matrix_offset[0] = 0;
    out->meta_matrix_offset[1] = mg;
    out->meta_matrix_offset[2] = 2 * mg;
    out->meta_per_expert = 2 * mg + md;
    out->planes_bytes = out->planes_per_expert * d->n_experts;
    out->meta_bytes = out->meta_per_expert * d->n_experts;
    out->rtable_bytes = static_cast<uint64_t>(d->n_experts) * B * 8;
    return DPA_OK;
}

size_t dpa_forward_workspace_size(const dpa_layer_desc* d, int max_tokens) {
    if (check_desc(d) != DPA_OK || max_tokens <= 0) return 0;
    return ws_layout(d, max_tokens).total;
}

dpa_status dpa_route(const dpa_layer_desc* d, const void* x, int n_tokens, const void* w_router,
                     int32_t* topk_idx, double* topk_gate, double* logits, void* ws, size_t ws_bytes,
                     void* stream) {
    const dpa_status st = check_desc(d);
    if (st != DPA_OK) return st;
    if (n_tokens <= 0 || n_tokens > 65535 || !x || !w_router || !topk_idx || !topk_gate || !ws)
        return DPA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(ws) || !aligned16(topk_idx) || !aligned16(topk_gate) ||
        (logits && !aligned16(logits)))
        return DPA_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(d, n_tokens);
    if (ws_bytes < L.total) return DPA_ERR_WORKSPACE;
    dpa::RouteArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.wr = static_cast<const uint16_t*>(w_router);
    a.T = n_tokens;
    a.E = d->n_experts;
    a.H = d->hidden;
    a.K = d->top_k;
    a.G = d->group;
    a.norm_topk = d->norm_topk;
    a.logits_user = logits;
    a.logits_ws = at<double>(ws, L.logits);
    a.idx = topk_idx;
    a.gate = topk_gate;
    a.counters = at<unsigned>(ws, L.counters);
    a.xdig = nullptr;
    a.hdr = at<dpa::WsHeader>(ws, L.hdr);
    set_route_stats(a, ws, L, n_tokens, d->n_experts);
    return dpa::launch_route(a, static_cast<cudaStream_t>(stream), num_sms_current()) == cudaSuccess ? DPA_OK
                                                                                                 : DPA_ERR_CUDA;
}

static dpa_status allocate_impl(const dpa_layer_desc* d, const double* rtable, const int32_t* idx,
                                const double* gate, int T, const double* target, uint8_t* k_out,
                                double* lambda_out, void* ws, const WsLayout& L, bool permute, cudaStream_t s,
                                bool gemm_tiles = false, int policy = DPA_ALLOC_LAGRANGE,
                                const double* threshold = nullptr, int vtiles_per_group = 1,
                                const uint8_t* expert_k = nullptr, const int* vgrid = nullptr,
                                const int* vnrb = nullptr, const uint8_t* expert_width = nullptr) {
    dpa::AllocArgs a{};
    a.policy = policy;
    a.threshold = threshold;
    a.expert_k = expert_k;
    a.expert_width = expert_width;
    a.rtable = rtable;
    a.idx = idx;
    a.gate = gate;
    a.target = target;
    a.T = T;
    a.K = d->top_k;
    a.E = d->n_experts;
    a.B = d->bits;
    a.kmin = d->kmin;
    a.kmax = d->kmax;
    a.k_out = k_out;
    a.lambda_out = lambda_out;
    a.cbuf = at<double>(ws, L.cbuf);
    a.do_permute = permute ? 1 : 0;
    a.pair_pos = at<int32_t>(ws, L.pairpos);
    a.gtiles = gemm_tiles ? at<int4>(ws, L.gtiles) : nullptr;
    a.pos_tok = gemm_tiles ? at<int32_t>(ws, L.postok) : nullptr;
    a.vrec = permute && !gemm_tiles ? at<int32_t>(ws, L.vrec) : nullptr;
    a.vtiles_per_group = vtiles_per_group;
    for (int j = 0; j < 2; ++j) {   // balanced CTA ranges of the two GEMV launches
        const bool use = a.vrec && vgrid && vgrid[j] > 0 && vgrid[j] <= kVpMaxGrid;
        a.vstart[j] = use ? at<int32_t>(ws, L.vstart) + j * (kVpMaxGrid + 1) : nullptr;
        a.vgrid[j] = use ? vgrid[j] : 0;
        a.vnrb[j] = use ? vnrb[j] : 0;
    }
    a.hdr = at<dpa::WsHeader>(ws, L.hdr);
    return dpa::launch_allocate(a, s, at<dpa::CoopSync>(ws, L.coop), num_sms_current()) == cudaSuccess ? DPA_OK
                                                                                                  : DPA_ERR_CUDA;
}

static bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// The policy and its scalar inputs: the budget policies read the target, the threshold policy
// the threshold.
static bool policy_inputs_ok(int policy, const double* target, const double* threshold, const uint8_t* expert_k) {
    if (policy == DPA_ALLOC_LAGRANGE || policy == DPA_ALLOC_UNIFORM) return target && aligned8(target);
    if (policy == DPA_ALLOC_THRESHOLD) return threshold && aligned8(threshold) && (!target || aligned8(target));
    if (policy == DPA_ALLOC_EXPERT_TABLE) return expert_k != nullptr && (!target || aligned8(target));
    return false;
}

dpa_status dpa_allocate_ex(const dpa_layer_desc* d, int policy, const double* rtable, const int32_t* topk_idx,
                           const double* topk_gate, int n_tokens, const double* target_bpw, const double* threshold,
                           const uint8_t* expert_k, uint8_t* k_out, double* lambda_out, void* ws, size_t ws_bytes,
                           void* stream) {
    const dpa_status st = check_desc(d);
    if (st != DPA_OK) return st;
    if (n_tokens <= 0 || n_tokens > 65535 || !topk_idx || !topk_gate || !k_out || !ws) return DPA_ERR_INVALID_ARG;
    if (!policy_inputs_ok(policy, target_bpw, threshold, expert_k)) return DPA_ERR_INVALID_ARG;
    if (policy == DPA_ALLOC_LAGRANGE && !rtable) return DPA_ERR_INVALID_ARG;
    if (!aligned16(ws) || (rtable && !aligned8(rtable)) || !aligned8(topk_gate) ||
        (reinterpret_cast<uintptr_t>(topk_idx) & 3) || (lambda_out && !aligned8(lambda_out)))
        return DPA_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(d, n_tokens);
    if (ws_bytes < L.total) return DPA_ERR_WORKSPACE;
    // the threshold and table policies read no target (the kernel never dereferences it then)
    return allocate_impl(d, rtable, topk_idx, topk_gate, n_tokens, target_bpw, k_out, lambda_out, ws, L, false,
                         static_cast<cudaStream_t>(stream), false, policy, threshold, 1, expert_k);
}

dpa_status dpa_allocate(const dpa_layer_desc* d, const double* rtable, const int32_t* topk_idx,
                        const double* topk_gate, int n_tokens, const double* target_bpw, uint8_t* k_out,
                        double* lambda_out, void* ws, size_t ws_bytes, void* stream) {
    return dpa_allocate_ex(d, DPA_ALLOC_LAGRANGE, rtable, topk_idx, topk_gate, n_tokens, target_bpw, nullptr, nullptr,
                           k_out, lambda_out, ws, ws_bytes, stream);
}

dpa_status dpa_profile_prefill(const dpa_layer_desc* d, const void* x, int n_tokens, const int32_t* topk_idx,
                               double* m, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
    const dpa_status st = check_desc(d);
    if (st != DPA_OK) return st;
    if (!x || n_tokens <= 0 || n_tokens > 65535 || !topk_idx || !m || !counts || !ws) return DPA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 1) || (reinterpret_cast<uintptr_t>(topk_idx) & 3) || !aligned8(m) ||
        (reinterpret_cast<uintptr_t>(counts) & 3) || !aligned16(ws))
        return DPA_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(d, 1).total) return DPA_ERR_WORKSPACE;
    dpa::ProfileArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.idx = topk_idx;
    a.T = n_tokens;
    a.H = d->hidden;
    a.K = d->top_k;
    a.E = d->n_experts;
    a.m = m;
    a.counts = counts;
    a.hdr = at<dpa::WsHeader>(ws, 0);
    return dpa::launch_profile(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DPA_OK : DPA_ERR_CUDA;
}

dpa_status dpa_solve_expert_rates(const dpa_layer_desc* d, const double* T, const double* m, const int32_t* counts,
                                  const double* target_bpw, uint8_t* k_table, double* lambda_out, void* ws,
                                  size_t ws_bytes, void* stream) {
    const dpa_status st = check_desc(d);
    if (st != DPA_OK) return st;
    if (!T || !m || !counts || !target_bpw || !k_table || !ws) return DPA_ERR_INVALID_ARG;
    if (!aligned8(T) || !aligned8(m) || (reinterpret_cast<uintptr_t>(counts) & 3) || !aligned8(target_bpw) ||
        (lambda_out && !aligned8(lambda_out)) || !aligned16(ws))
        return DPA_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(d, 1).total) return DPA_ERR_WORKSPACE;
    dpa::RatesArgs a{};
    a.tdist = T;
    a.m = m;
    a.counts = counts;
    a.target = target_bpw;
    a.E = d->n_experts;
    a.B = d->bits;
    a.H = d->hidden;
    a.kmin = d->kmin;
    a.kmax = d->kmax;
    a.k_table = k_table;
    a.lambda_out = lambda_out;
    a.hdr = at<dpa::WsHeader>(ws, 0);
    return dpa::launch_solve_rates(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DPA_OK : DPA_ERR_CUDA;
}

dpa_status dpa_calibrate_threshold(const dpa_layer_desc* d, const double* scores, int n_scores,
                                   const double* target_bpw, double* threshold_out, void* ws, size_t ws_bytes,
                                   void* stream) {
    const dpa_status st = check_desc(d);
    if (st != DPA_OK) return st;
    if (!scores || n_scores <= 0 || n_scores > (1 << 26) || !target_bpw || !threshold_out || !ws)
        return DPA_ERR_INVALID_ARG;
    if (!aligned8(scores) || !aligned8(target_bpw) || !aligned8(threshold_out) || !aligned16(ws))
        return DPA_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(d, 1).total) return DPA_ERR_WORKSPACE;
    dpa::CalibArgs a{};
    a.scores = scores;
    a.n = n_scores;
    a.kmin = d->kmin;
    a.kmax = d->kmax;
    a.target = target_bpw;
    a.threshold_out = threshold_out;
    a.hdr = at<dpa::WsHeader>(ws, 0);
    return dpa::launch_calibrate(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DPA_OK : DPA_ERR_CUDA;
}

dpa_status dpa_moe_forward(const dpa_layer_desc* d, const dpa_layer_weights* w, const void* x, int n_tokens,
                           const double* target_bpw, void* y, dpa_aux* aux, void* ws, size_t ws_bytes,
                           void* stream) {
    const dpa_status st = check_desc(d);
    if (st != DPA_OK) return st;
    if (!w || !x || !y || !ws || !target_bpw || n_tokens <= 0 || n_tokens > 65535) return DPA_ERR_INVALID_ARG;
    if (!w->planes || !w->meta || !w->rtable || !w->w_router) return DPA_ERR_INVALID_ARG;
    if (d->n_shared > 0 && (!w->shared_gate || !w->shared_up || !w->shared_down)) return DPA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(ws) || !aligned16(w->planes) || !aligned16(w->meta) ||
        !aligned16(w->w_router) || (reinterpret_cast<uintptr_t>(w->rtable) & 7) ||
        (reinterpret_cast<uintptr_t>(target_bpw) & 7))
        return DPA_ERR_INVALID_ARG;
    if (d->n_shared > 0 && (!aligned16(w->shared_gate) || !aligned16(w->shared_up) || !aligned16(w->shared_down)))
        return DPA_ERR_INVALID_ARG;
    if (aux && aux->pair_out && !aligned16(aux->pair_out)) return DPA_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(d, n_tokens);
    if (ws_bytes < L.total) return DPA_ERR_WORKSPACE;
    dpa_sizes sz;
    dpa_encoded_sizes(d, &sz);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = n_tokens, K = d->top_k;
    const int path = aux ? aux->expert_path : DPA_PATH_AUTO;
    if (path < DPA_PATH_AUTO || path > DPA_PATH_TC) return DPA_ERR_INVALID_ARG;
    const int policy = aux ? aux->alloc_policy : DPA_ALLOC_LAGRANGE;
    const double* threshold = aux ? aux->threshold : nullptr;
    const uint8_t* expert_k = aux ? aux->expert_k : nullptr;
    if (!policy_inputs_ok(policy, target_bpw, threshold, expert_k)) return DPA_ERR_INVALID_ARG;
    const bool tc_shape = d->format == DPA_FMT_UNIFORM && d->hidden % 256 == 0 && d->inter % 256 == 0 &&
                          (d->group & (d->group - 1)) == 0;   // scale groups of 64 * 2^n inputs
    const bool compact = w->expert_width != nullptr || w->expert_offsets != nullptr;
    if (compact && !(w->expert_width && w->expert_offsets)) return DPA_ERR_INVALID_ARG;
    if (path == DPA_PATH_TC && (!tc_shape || compact)) return DPA_ERR_UNSUPPORTED;
    const bool use_tc = path == DPA_PATH_TC ||
                        (path == DPA_PATH_AUTO && tc_shape && !compact &&
                         static_cast<long long>(T) * K >= static_cast<long long>(DPA_TC_MIN_PAIRS_PER_EXPERT) * d->n_experts);

    int32_t* idx = (aux && aux->topk_idx) ? aux->topk_idx : at<int32_t>(ws, L.idx);
    double* gate = (aux && aux->topk_gate) ? aux->topk_gate : at<double>(ws, L.gate);
    uint8_t* kk = (aux && aux->k) ? aux->k : at<uint8_t>(ws, L.k);
    double* lam = (aux && aux->lambda) ? aux->lambda : at<double>(ws, L.lambda);
    dpa::WsHeader* hdr = at<dpa::WsHeader>(ws, L.hdr);

    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (aux) cudaStreamIsCapturing(s, &cap);
    const StageMarks mark{aux, s, cap};
    mark(0);
    // 1. route (+ fixed-point digits of x)
    dpa::RouteArgs ra{};
    ra.x = static_cast<const uint16_t*>(x);
    ra.wr = static_cast<const uint16_t*>(w->w_router);
    ra.T = T;
    ra.E = d->n_experts;
    ra.H = d->hidden;
    ra.K = K;
    ra.G = d->group;
    ra.norm_topk = d->norm_topk;
    ra.logits_user = nullptr;
    ra.logits_ws = at<double>(ws, L.logits);
    ra.idx = idx;
    ra.gate = gate;
    ra.counters = at<unsigned>(ws, L.counters);
    ra.xdig = use_tc ? nullptr : at<int8_t>(ws, L.xdig);   // the tensor-core path reads x directly
    ra.xscl = at<float>(ws, L.xscl);
    ra.xfsx = at<float>(ws, L.xfsx);
    ra.hdr = hdr;
    set_route_stats(ra, ws, L, T, d->n_experts);
    if (dpa::launch_route(ra, s, num_sms_current()) != cudaSuccess) return DPA_ERR_CUDA;
    mark(1);

    // 2. allocate + group pairs by (expert, k)
    // the expert GEMV's variant: one token per expert (batch 1) runs the small-batch kernels;
    // otherwise token groups of up to two 4-pair tiles, where their staging fits
    // token groups of the expert GEMV: two 4-pair tiles where the group slots fit, else one
    const int tpg = dpa::vp_tiles_per_group(d->hidden, d->inter, d->group, d->format, d->bits);
    // the two GEMV launches (decode path): their grids and row blocks per record, for which the
    // allocation writes work-balanced CTA ranges
    dpa::VpArgs va_gu{}, va_dn{};
    int vgrid[2] = {0, 0}, vnrb[2] = {0, 0};
    if (!use_tc) {
        const int nsm = num_sms_current();
        va_gu = vp_launch_args(d, w, sz, ws, L, T, tpg, false);
        va_dn = vp_launch_args(d, w, sz, ws, L, T, tpg, true);
        vgrid[0] = dpa::vp_grid(va_gu, nsm);
        vgrid[1] = dpa::vp_grid(va_dn, nsm);
        vnrb[0] = va_gu.R / dpa::vp_rows_per_item(va_gu);
        vnrb[1] = va_dn.R / dpa::vp_rows_per_item(va_dn);
    }
    dpa_status st2 = allocate_impl(d, w->rtable, idx, gate, T, target_bpw, kk, lam, ws, L, true, s, use_tc, policy,
                                   threshold, tpg, expert_k, vgrid, vnrb, w->expert_width);
    if (st2 != DPA_OK) return st2;
    mark(2);

    // 3. dense shared experts
    if (d->n_shared > 0) {
        dpa::SharedArgs sa{};
        sa.x = static_cast<const uint16_t*>(x);
        sa.wg = static_cast<const uint16_t*>(w->shared_gate);
        sa.wu = static_cast<const uint16_t*>(w->shared_up);
        sa.wd = static_cast<const uint16_t*>(w->shared_down);
        sa.h = at<float>(ws, L.sh_h);
        sa.out = at<float>(ws, L.sh_out);
        sa.T = T;
        sa.S = d->n_shared;
        sa.H = d->hidden;
        sa.I = d->inter;
        if (dpa::launch_shared(sa, s) != cudaSuccess) return DPA_ERR_CUDA;
    }
    mark(3);

    // 4. variable-plane expert FFN
    const int sms = num_sms_current();
    if (use_tc) {
        dpa::GemmArgs ta{};
        ta.planes = static_cast<const uint8_t*>(w->planes);
        ta.meta = static_cast<const uint8_t*>(w->meta);
        ta.planes_per_expert = sz.planes_per_expert;
        ta.meta_per_expert = sz.meta_per_expert;
        for (int m = 0; m < 3; ++m) {
            ta.planes_mat_off[m] = sz.planes_matrix_offset[m];
            ta.meta_mat_off[m] = sz.meta_matrix_offset[m];
        }
        ta.H = d->hidden;
        ta.I = d->inter;
        ta.B = d->bits;
        ta.G = d->group;
        ta.T = T;
        ta.P = T * K;
        ta.gtiles = at<int4>(ws, L.gtiles);
        ta.pos_tok = at<int32_t>(ws, L.postok);
        ta.x = static_cast<const uint16_t*>(x);
        ta.xperm = at<uint16_t>(ws, L.xperm);
        ta.E = d->n_experts;
        ta.hbuf = at<uint16_t>(ws, L.h);
        ta.out_pair = at<float>(ws, L.out_pair);
        ta.hdr = hdr;
        if (dpa::launch_permute_rows(ta, s) != cudaSuccess) return DPA_ERR_CUDA;
        if (dpa::launch_gemm_gateup(ta, s, sms) != cudaSuccess) return DPA_ERR_CUDA;
        mark(4);
        if (dpa::launch_gemm_down(ta, s, sms) != cudaSuccess) return DPA_ERR_CUDA;
        mark(5);
        return combine_stage(d, w, gate, T, aux, y, ws, L, hdr, s, mark);
    }
    const int P = T * K;
    // gate and up with SwiGLU: x digits by token -> h [P][I]
    dpa::VpArgs va = va_gu;
    va.vstart = vgrid[0] > 0 && vgrid[0] <= kVpMaxGrid ? at<int32_t>(ws, L.vstart) : nullptr;
    va.vgrid = vgrid[0];
    if (dpa::launch_vp_gemv(va, s, sms) != cudaSuccess) return DPA_ERR_CUDA;
    mark(4);
    // digits of h, then down -> per-pair outputs [P][H]
    dpa::DigitArgs da{};
    da.x16 = nullptr;
    da.x32 = at<float>(ws, L.h);
    da.rows = P;
    da.K = d->inter;
    da.G = d->group;
    da.dig = at<int8_t>(ws, L.hdig);
    da.dscl = at<float>(ws, L.hscl);
    da.dfsx = at<float>(ws, L.hfsx);
    if (dpa::launch_digits(da, s) != cudaSuccess) return DPA_ERR_CUDA;
    va = va_dn;
    va.vstart = vgrid[1] > 0 && vgrid[1] <= kVpMaxGrid ? at<int32_t>(ws, L.vstart) + (kVpMaxGrid + 1) : nullptr;
    va.vgrid = vgrid[1];
    if (dpa::launch_vp_gemv(va, s, sms) != cudaSuccess) return DPA_ERR_CUDA;
    mark(5);
    return combine_stage(d, w, gate, T, aux, y, ws, L, hdr, s, mark);
}

dpa_status dpa_residual_rmsnorm(const void* y, float* h, int n_tokens, int hidden, void* x, void* stream) {
    if (!h || !x || n_tokens <= 0 || n_tokens > 2147483647 || hidden <= 0 || hidden % 4) return DPA_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(x) || (y && !aligned16(y))) return DPA_ERR_INVALID_ARG;
    return dpa::launch_residual_rmsnorm(static_cast<const uint16_t*>(y), h, static_cast<uint16_t*>(x), n_tokens, hidden,
                                        1e-6f, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? DPA_OK
               : DPA_ERR_CUDA;
}

dpa_status dpa_stream_prefixes(const dpa_layer_desc* d, const void* host_planes, const void* host_meta,
                               const int32_t* experts, const uint8_t* kplanes, int n, void* dev_planes, void* dev_meta,
                               uint64_t* bytes_out, void* stream) {
    const dpa_status st = check_desc(d);
    if (st != DPA_OK) return st;
    if (!host_planes || !host_meta || !experts || !kplanes || n < 0 || !dev_planes || !dev_meta)
        return DPA_ERR_INVALID_ARG;
    dpa_sizes sz;
    dpa_encoded_sizes(d, &sz);
    for (int i = 0; i < n; ++i)
        if (experts[i] < 0 || experts[i] >= d->n_experts || kplanes[i] < 1 || kplanes[i] > d->bits)
            return DPA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint8_t* hp = static_cast<const uint8_t*>(host_planes);
    const uint8_t* hm = static_cast<const uint8_t*>(host_meta);
    uint8_t* dp = static_cast<uint8_t*>(dev_planes);
    uint8_t* dm = static_cast<uint8_t*>(dev_meta);
    const uint64_t H = d->hidden, I = d->inter, G = d->group, B = d->bits;
    uint64_t total = 0;
    for (int i = 0; i < n; ++i) {
        const uint64_t e = static_cast<uint64_t>(experts[i]), k = kplanes[i];
        for (int m = 0; m < 3; ++m) {
            // the first k planes of a matrix are one contiguous prefix of its bytes
            const uint64_t plane_bytes = H * I / 8;
            const uint64_t off = e * sz.planes_per_expert + sz.planes_matrix_offset[m];
            if (cudaMemcpyAsync(dp + off, hp + off, k * plane_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
                return DPA_ERR_CUDA;
            total += k * plane_bytes;
            if (d->format == DPA_FMT_BCQ) {   // the first k planes' alphas, a prefix per matrix too
                const uint64_t R = m == 2 ? H : I, C = m == 2 ? I : H;
                const uint64_t moff = e * sz.meta_per_expert + sz.meta_matrix_offset[m];
                const uint64_t abytes = k * R * (C / G) * 2;
                if (cudaMemcpyAsync(dm + moff, hm + moff, abytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
                    return DPA_ERR_CUDA;
                total += abytes;
            }
        }
        if (d->format == DPA_FMT_UNIFORM) {   // scales and zeros serve every k: the expert's whole block
            const uint64_t moff = e * sz.meta_per_expert;
            if (cudaMemcpyAsync(dm + moff, hm + moff, sz.meta_per_expert, cudaMemcpyHostToDevice, s) != cudaSuccess)
                return DPA_ERR_CUDA;
            total += sz.meta_per_expert;
        }
    }
    (void)B;
    if (bytes_out) *bytes_out = total;
    return DPA_OK;
}

dpa_status dpa_device_status(void* ws, void* stream) {
    if (!ws) return DPA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return DPA_ERR_CUDA;
    uint32_t v[2] = {0, 0};
    if (cudaMemcpy(v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return DPA_ERR_CUDA;
    if (v[0] != 0) {
        const uint32_t zero[2] = {0, 0};
        if (cudaMemcpy(ws, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return DPA_ERR_CUDA;
    }
    return static_cast<dpa_status>(v[0]);
}

}  // extern "C"
