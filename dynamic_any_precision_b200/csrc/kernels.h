// Launch interfaces of the device kernels (internal to the library).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace dpa {

struct RouteArgs {
    const uint16_t* x;        // [T][H] bf16
    const uint16_t* wr;       // [E][H] bf16
    int T, E, H, K, G, norm_topk;
    double* logits_user;      // [T][E] or nullptr
    double* logits_ws;        // [T][E] workspace copy
    int32_t* idx;             // [T][K]
    double* gate;             // [T][K]
    unsigned* counters;       // [T] zero between calls
    int8_t* xdig;             // [T][3][H] or nullptr (digits not needed)
    int32_t* xexp;            // [T][H/G]
    int32_t* xsum;            // [T][H/G]
    WsHeader* hdr;
    int wpe;                  // warps per expert (set by the launcher)
    // large-batch path (nullptr: always the per-logit kernel): per-row exactness statistics
    int16_t* lsb_x;           // [T][H/64] lowest set bit over each 64-input block's nonzero elements
    double* n2_x;             // [T] sum of squares
    int16_t* lsb_w;           // [E][H/64]
    double* n2_w;             // [E]
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream, int sms = 148);

struct AllocArgs {
    const double* rtable;     // [E][B]
    const int32_t* idx;       // [T][K]
    const double* gate;       // [T][K]
    const double* target;     // device scalar
    int T, K, E, B, kmin, kmax;
    uint8_t* k_out;           // [T][K]
    double* lambda_out;       // scalar or nullptr
    double* cbuf;             // [P][nk] workspace
    // grouping outputs (do_permute)
    int do_permute;
    int32_t* pair_pos;        // [P] position of each pair in the (expert, k)-grouped order
    int4* exp_desc;           // [E][2] per active expert: {expert, kmax, n_tiles, first tile}, first tile
    int4* tiles;              // [P + E*nk] two-token tiles: {k, posA, posB, tokA | tokB << 16}
    int k_given;              // 1: k_out already holds the plane counts (grid-wide bisection ran)
    int4* gtiles;             // nullptr, or [P/kGemmTileTokens + E*nk] GEMM token tiles {e, k, pos0, n}
    int32_t* pos_tok;         // nullptr, or [P] token of each grouped position
    WsHeader* hdr;
    int policy;               // DPA_ALLOC_LAGRANGE, DPA_ALLOC_UNIFORM or DPA_ALLOC_THRESHOLD
    const double* threshold;  // device scalar (DPA_ALLOC_THRESHOLD)
};
// Counters of the grid-wide bisection (zeroed by the launcher before every call).
constexpr int kCoopRoundsMax = 16;
struct CoopSync {
    unsigned barrier;
    unsigned bad;
    unsigned long long mx_bits;
    int counts[kCoopRoundsMax][64][32];   // one 128-byte line per node: CTAs' atomics do not queue on one line
};
// coop: workspace counters for the grid-wide bisection of large batches (nullptr: single CTA).
cudaError_t launch_allocate(const AllocArgs& a, cudaStream_t stream, CoopSync* coop = nullptr, int sms = 0);
size_t allocate_smem_bytes(int P, int E, int nk);
int allocate_threads(int P);

// Threshold calibration of the score-threshold policy: 64 bisection steps over n scores.
struct CalibArgs {
    const double* scores;     // [n]
    int n, kmin, kmax;
    const double* target;     // device scalar
    double* threshold_out;    // device scalar
    WsHeader* hdr;
};
cudaError_t launch_calibrate(const CalibArgs& a, cudaStream_t stream);

// Prefill expert FFN on tcgen05: grouped GEMMs over the GEMM token tiles of the allocation.
struct GemmArgs {
    const uint8_t* planes;    // encoded layer (uniform format)
    const uint8_t* meta;
    uint64_t planes_per_expert, meta_per_expert;
    uint64_t planes_mat_off[3], meta_mat_off[3];
    int H, I, B, G;
    int T, P;                 // tokens, routed pairs (rows of x and of hbuf)
    const int4* gtiles;       // {e, k, pos0, n}, count in hdr->n_gtiles
    const int32_t* pos_tok;   // [P] token of each grouped position
    const uint16_t* x;        // [T][H] bf16 activations
    uint16_t* xperm;          // [P][H] bf16 activations in grouped pair order (written by the permute)
    int E;
    uint16_t* hbuf;           // [P][I] fp16 SwiGLU outputs, grouped order
    float* out_pair;          // [P][H] per-pair expert outputs, grouped order
    WsHeader* hdr;
};
cudaError_t launch_permute_rows(const GemmArgs& a, cudaStream_t stream);
cudaError_t launch_gemm_gateup(const GemmArgs& a, cudaStream_t stream, int sms);
cudaError_t launch_gemm_down(const GemmArgs& a, cudaStream_t stream, int sms);
size_t gemm_tc_smem_bytes();

struct GemvArgs {
    const uint8_t* planes;    // encoded layer
    const uint8_t* meta;
    uint64_t planes_per_expert, meta_per_expert;
    uint64_t planes_mat_off[3], meta_mat_off[3];
    int E, H, I, K, B, G, kmin, kmax, fmt;
    const int4* exp_desc;     // per active expert [2]: {expert, kmax, n_tiles, first tile}, first tile
    const int4* tiles;        // {k, posA, posB, tokA | tokB << 16}
    const int8_t* xdig;       // [T][3][H]
    const int32_t* xexp;      // [T][H/G]
    const int32_t* xsum;      // [T][H/G]
    float* h;                 // [P][I] by sorted position
    float* out_pair;          // [P][H] by sorted position
    int8_t* hdig;             // [P][3][I] digits of h (multi-token down kernel)
    int32_t* hexp;            // [P][I/G]
    int32_t* hsum;            // [P][I/G]
    int P;                    // routed pairs
    WsHeader* hdr;
    int max_items;            // upper bound of active experts (host-known)
    int max_tokens_per_expert;  // host-known bound (selects the tile count per pass)
};
cudaError_t launch_gateup(const GemvArgs& a, cudaStream_t stream, int num_sms);
// Dynamic shared memory a GEMV work item may stage. The single-pass (one- and two-token)
// kernels must fit for a layer to be accepted; the multi-token kernels run only where they fit
// too, the single-pass ones (one tile per pass) elsewhere.
constexpr size_t kGemvMaxSmem = 200 * 1024;
size_t gateup_smem_bytes(const GemvArgs& a);   // one CTA of the single-pass gate/up kernel
size_t down_smem_bytes(const GemvArgs& a);     // one CTA of the single-pass down kernel
cudaError_t launch_down(const GemvArgs& a, cudaStream_t stream, int num_sms);

struct CombineArgs {
    const float* out_pair;    // [P][H] by sorted position
    const int32_t* pair_pos;  // [P]
    const double* gate;       // [T][K]
    const float* shared_out;  // [T][H] or nullptr
    float* pair_out_user;     // [T][K][H] diagnostic copy or nullptr
    uint16_t* y;              // [T][H] bf16
    int T, K, H;
    WsHeader* hdr;
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream);

struct SharedArgs {
    const uint16_t* x;        // [T][H] bf16
    const uint16_t* wg;       // [S][I][H]
    const uint16_t* wu;
    const uint16_t* wd;       // [S][H][I]
    float* h;                 // [T][S][I] workspace
    float* out;               // [T][H]
    int T, S, H, I;
};
cudaError_t launch_shared(const SharedArgs& a, cudaStream_t stream);

cudaError_t launch_residual_rmsnorm(const uint16_t* y, float* h, uint16_t* x, int T, int H, float eps,
                                    cudaStream_t stream);

}  // namespace dpa
