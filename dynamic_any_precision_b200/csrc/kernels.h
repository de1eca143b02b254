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
    int8_t* xdig;             // [T][2][H] activation digits for the expert GEMV, or nullptr
    float* xscl;              // [T][ngp] group scales 2^(E-14) (ngp = H/G rounded up to 4)
    float* xfsx;              // [T][ngp] group sums of the fixed-point values times the scale
    WsHeader* hdr;
    int wpe;                  // warps per expert (set by the launcher)
    // large-batch path (nullptr: always the per-logit kernel): per-row exactness statistics
    int16_t* lsb_x;           // [T][H/64] lowest set bit over each 64-input block's nonzero elements
    int16_t* hb_x;            // [T][H/64] h with |x_b| < 2^h (Euclidean norm of the block)
    double* n2_x;             // [T] sum of squares
    int16_t* lsb_w;           // [E][H/64]
    int16_t* hb_w;            // [E][H/64]
    double* n2_w;             // [E]
    double* part;             // [ks][T][E] slice sums of the tiled logits
    int ks;                   // input slices (set by the launcher)
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t stream, int sms = 148);

// Tiling of the large-batch logits: token x expert CTA tiles, input slices to fill the SMs.
struct RouteTiling {
    int TT, TE, gx, gy, ks, kslice;
};
constexpr int kRouteMaxSms = 256;   // the partial-sum buffer is sized for up to this many SMs
RouteTiling route_tiling(int T, int E, int H, int sms);
bool route_tiled_path(int T, int H);
// doubles of the slice-sum buffer the tiled path needs for T tokens (0: the per-logit path)
size_t route_partial_doubles(int T, int E, int H);

// A token group of the expert GEMV: [0] expert, [1] kmax over the group, [2] tiles (<= 2),
// [4 + t] plane count of tile t, [6 + t] pairs in tile t (<= 4), [8 + 4t + q] grouped position
// (output row) of pair q of tile t, [16 + 4t + q] its token; unused slots hold -1.
constexpr int kVRecInts = 32;

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
    int k_given;              // 1: k_out already holds the plane counts (grid-wide bisection ran)
    int4* gtiles;             // nullptr, or [P/kGemmTileTokens + E*nk] GEMM token tiles {e, k, pos0, n}
    int32_t* pos_tok;         // nullptr, or [P] token of each grouped position
    WsHeader* hdr;
    int policy;               // DPA_ALLOC_LAGRANGE, DPA_ALLOC_UNIFORM or DPA_ALLOC_THRESHOLD
    const double* threshold;  // device scalar (DPA_ALLOC_THRESHOLD)
    // work list of the pipelined expert GEMV (nullptr: not written): token groups of up to
    // vtiles_per_group (<= 2) tiles of up to 4 pairs of one (expert, k) class, as records of
    // kVRecInts ints (see kVRec*); count in hdr->n_vgroups
    int32_t* vrec;            // [P/4 + E*nk][kVRecInts]
    int vtiles_per_group;
    // per GEMV launch j (0: gate/up, 1: down), unless vstart[j] is nullptr: the first item of each
    // of its vgrid[j] CTAs over items (record, row block; vnrb[j] row blocks per record), with
    // equal shares of the estimated work; vstart[j][vgrid[j]] = the item count
    int32_t* vstart[2];
    int vgrid[2], vnrb[2];
    const uint8_t* expert_k;  // [E] plane count per expert (DPA_ALLOC_EXPERT_TABLE)
    const uint8_t* expert_width;   // nullptr, or [E] stored planes per expert: no pair reads more
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
size_t allocate_smem_bytes(int P, int E, int nk, bool recs);
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

// Workload profile of a prefill and the per-expert read rates solved from it.
struct ProfileArgs {
    const uint16_t* x;        // [T][H] bf16 prefill activations
    const int32_t* idx;       // [T][K] routed experts
    int T, H, K, E;
    double* m;                // [H] mean square per input channel
    int32_t* counts;          // [E] routed pairs per expert
    WsHeader* hdr;
};
cudaError_t launch_profile(const ProfileArgs& a, cudaStream_t stream);
struct RatesArgs {
    const double* tdist;      // [E][B][H] distortion tensor
    const double* m;          // [H]
    const int32_t* counts;    // [E]
    const double* target;     // device scalar
    int E, B, H, kmin, kmax;
    uint8_t* k_table;         // [E]
    double* lambda_out;       // scalar or nullptr
    WsHeader* hdr;
};
cudaError_t launch_solve_rates(const RatesArgs& a, cudaStream_t stream);
size_t rates_smem_bytes(int E, int nk);

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

// Pipelined variable-plane expert GEMV (decode batches): one launch computes either gate and up
// with the SwiGLU epilogue (nmat = 2: out = h [P][R], R = inter) or down (nmat = 1: out =
// per-pair outputs [P][R], R = hidden) for every (token group, row block) item.
struct VpArgs {
    const uint8_t* planes;    // encoded layer
    const uint8_t* meta;
    uint64_t planes_per_expert, meta_per_expert;
    uint64_t planes_mat_off[3], meta_mat_off[3];
    int fmt, B, G;
    int R, K;                 // rows and columns of each matrix of this launch
    int mat0, nmat;           // first matrix (0: gate, up; 2: down) and the matrix count
    int tiles_per_group;      // 1 or 2 (the allocation's grouping)
    const int32_t* vrec;      // token group records [n_vgroups][kVRecInts], count in hdr->n_vgroups
    const int8_t* dig;        // activation digit rows [rows][2][K] (permuted 64-column blocks)
    const float* dscl;        // [rows][ngp] group scales 2^(E-14)
    const float* dfsx;        // [rows][ngp] group sums of the fixed-point values times the scale
    int dig_by_token;         // 1: the digit row of a pair is its token (x); 0: its position (h)
    float* out;               // [P][R] by grouped position
    WsHeader* hdr;
    int max_groups;           // host bound of the token groups
    const uint64_t* expert_off;   // nullptr (full layout), or [E][2] byte offsets of each expert's
                                  // planes and scale data in the compact layer of stored widths
    const uint8_t* expert_width;  // [E] stored planes per expert (with expert_off)
    const int32_t* vstart;    // nullptr (equal item counts per CTA), or [grid + 1] first item of each
                              // CTA, balanced by estimated work (written by the allocation)
    int vgrid;                // the grid vstart was written for (used only when the launch matches)
};
cudaError_t launch_vp_gemv(const VpArgs& a, cudaStream_t stream, int sms);
// The launch geometry of a variant, as launch_vp_gemv will use it: CTAs and rows per item.
int vp_grid(const VpArgs& a, int sms);
int vp_rows_per_item(const VpArgs& a);
// tiles per token group the layer's shapes allow (2 where the group slots fit, else 1)
int vp_tiles_per_group(int K_gateup, int K_down, int G, int fmt, int B);
// dynamic shared memory of one CTA of a variant
size_t vp_smem_bytes(int K, int G, int fmt, int B, int nmat, int tiles_per_group);
constexpr size_t kVpMaxSmem = 227 * 1024;

// Fixed-point digits of activation rows (x as bf16, or h as fp32), per group of G columns:
// X = rint(v * 2^(14 - E)) with |v| < 2^E, as digits d0 + 256 d1 in rows [rows][2][K] with each
// 64-column block permuted for the B operand; per group the scale 2^(E-14) and the scaled sum
// 2^(E-14) sum_j X_j (both exact in fp32), [rows][ngp], ngp = K/G rounded up to a multiple of 4.
struct DigitArgs {
    const uint16_t* x16;      // bf16 rows or nullptr
    const float* x32;         // fp32 rows (when x16 is nullptr)
    int rows, K, G;
    int8_t* dig;
    float* dscl;
    float* dfsx;
};
cudaError_t launch_digits(const DigitArgs& d, cudaStream_t stream);

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
