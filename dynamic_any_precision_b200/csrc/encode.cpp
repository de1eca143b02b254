// Offline encoder of routed expert weights into prefix-decodable bitplanes (host C++).
//
// DPA-MoE: A Runtime Precision Control Framework for MoE Inference, Abstract: each expert's
// FFN weights are encoded so that every leading run of chunks decodes on its own, all runs
// sharing one scale (the page names the format SharedScale AnyBCQ), and each expert's
// reconstruction error is measured ahead of time.
// MatMoE (review, "Core Contribution"): weights are kept as bitplanes, and the low-bit prefix
// and the full code use the same quantisation parameters.
// DuoRate, Abstract: a single stored copy whose prefix can be read at any rate, plus a
// precomputed table of distortions.
//
// Build with -ffp-contract=off and without fast-math: every fp64 operation below is one IEEE
// round-to-nearest operation, so the codes, scales and residual sums are reproducible.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

#include "dpa.h"
#include "layout.h"

namespace {

// ---- fp16 <-> fp64 (round to nearest, ties to even, gradual underflow) ----
uint16_t f64_to_f16_bits(double v) {
    uint64_t b;
    std::memcpy(&b, &v, 8);
    const uint16_t sign = static_cast<uint16_t>((b >> 48) & 0x8000u);
    const int exp = static_cast<int>((b >> 52) & 0x7FF);
    uint64_t man = b & ((1ull << 52) - 1);
    if (exp == 0x7FF) return sign | 0x7C00u | (man ? 0x200u : 0u);
    if (exp == 0 && man == 0) return sign;
    // value = 1.man * 2^(exp-1023) (fp64 subnormals are far below fp16's range -> 0)
    int e = exp - 1023;
    if (exp == 0) return sign;
    uint64_t sig = man | (1ull << 52);          // 53-bit significand
    int shift;                                   // bits of sig to drop
    uint16_t hexp;
    if (e >= -14) {                              // normal fp16 candidate
        shift = 52 - 10;
        hexp = static_cast<uint16_t>(e + 15);
    } else {                                     // subnormal fp16: unit 2^-24
        shift = 52 - 10 + (-14 - e);
        hexp = 0;
        if (shift > 63) return sign;
    }
    uint64_t keep = sig >> shift;
    uint64_t rem = sig & ((1ull << shift) - 1);
    uint64_t half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (keep & 1))) keep += 1;
    uint32_t out;
    if (hexp == 0) {
        out = static_cast<uint32_t>(keep);       // may carry into the smallest normal: fine
    } else {
        if (keep >> 11) { keep >>= 1; hexp += 1; }
        if (hexp >= 31) return sign | 0x7C00u;   // overflow -> inf
        out = (static_cast<uint32_t>(hexp) << 10) | static_cast<uint32_t>(keep & 0x3FF);
    }
    return sign | static_cast<uint16_t>(out);
}

double f16_bits_to_f64(uint16_t h) {
    const int sign = (h >> 15) & 1;
    const int exp = (h >> 10) & 0x1F;
    const int man = h & 0x3FF;
    double v;
    if (exp == 0) v = std::ldexp(static_cast<double>(man), -24);
    else if (exp == 31) v = man ? NAN : INFINITY;
    else v = std::ldexp(static_cast<double>(man | 0x400), exp - 25);
    return sign ? -v : v;
}

struct Mat {
    const float* w;   // [R][C]
    int R, C;
};

// Place the code bits of weight (row, col) of one matrix into its planes.
inline void set_code(uint32_t* mat_planes, uint64_t plane_words, int R, int C, int row, int col,
                     unsigned code, int B, bool uniform) {
    for (int p = 0; p < B; ++p) {
        if ((code >> (B - 1 - p)) & 1u) {
            const dpa_layout::BitPos bp = dpa_layout::bit_position(C, row, col, p, B, uniform);
            mat_planes[static_cast<uint64_t>(p) * plane_words + bp.word] |= (1u << bp.bit);
        }
    }
    (void)R;
}

// The code of weight (row, col) read back from its planes.
inline unsigned get_code(const uint32_t* mat_planes, uint64_t plane_words, int C, int row, int col, int B,
                         bool uniform) {
    unsigned code = 0;
    for (int p = 0; p < B; ++p) {
        const dpa_layout::BitPos bp = dpa_layout::bit_position(C, row, col, p, B, uniform);
        code |= ((mat_planes[static_cast<uint64_t>(p) * plane_words + bp.word] >> bp.bit) & 1u) << (B - 1 - p);
    }
    return code;
}

struct EncodeJob {
    const dpa_layer_desc* d;
    dpa_sizes sz;
    const float* wg; const float* wu; const float* wd;
    uint8_t* planes; uint8_t* meta; double* rtable;
    int e_begin;
};

// Uniform asymmetric codes of one matrix; accumulates (w - w_k)^2 into acc[k-1].
bool encode_uniform_matrix(const Mat& m, int B, int G, uint32_t* mat_planes, uint16_t* mat_meta,
                           double* acc) {
    const double qmax = static_cast<double>((1 << B) - 1);
    const int ng = m.C / G;
    const uint64_t plane_words = static_cast<uint64_t>(m.R) * m.C / 32;
    std::vector<double> s_row(ng), z_row(ng);
    std::vector<unsigned> q_row(m.C);
    for (int r = 0; r < m.R; ++r) {
        const float* wr = m.w + static_cast<uint64_t>(r) * m.C;
        for (int g = 0; g < ng; ++g) {
            double lo = wr[g * G], hi = wr[g * G];
            for (int j = 1; j < G; ++j) {
                const double v = wr[g * G + j];
                lo = v < lo ? v : lo;
                hi = v > hi ? v : hi;
            }
            const double range = hi - lo;
            const double s_raw = range / qmax;
            uint16_t sb = f64_to_f16_bits(s_raw);
            double s = f16_bits_to_f64(sb);
            if (s == 0.0) { sb = 0x3C00u; s = 1.0; }
            if (!std::isfinite(s)) return false;
            double z = std::nearbyint(-lo / s);
            z = z < 0.0 ? 0.0 : (z > qmax ? qmax : z);
            s_row[g] = s;
            z_row[g] = z;
            mat_meta[(static_cast<uint64_t>(r) * ng + g) * 2 + 0] = sb;
            mat_meta[(static_cast<uint64_t>(r) * ng + g) * 2 + 1] = f64_to_f16_bits(z);
            for (int j = 0; j < G; ++j) {
                const double v = wr[g * G + j];
                double q = std::nearbyint(v / s) + z;
                q = q < 0.0 ? 0.0 : (q > qmax ? qmax : q);
                q_row[g * G + j] = static_cast<unsigned>(q);
            }
        }
        for (int c = 0; c < m.C; ++c) {
            set_code(mat_planes, plane_words, m.R, m.C, r, c, q_row[c], B, true);
            const double w = wr[c];
            const double s = s_row[c / G], z = z_row[c / G];
            for (int k = 1; k <= B; ++k) {
                const int dsh = B - k;
                const double qk = static_cast<double>(q_row[c] >> dsh);
                const double pw = static_cast<double>(1u << dsh);
                const double qhat = qk * pw + (pw - 1.0) / 2.0;
                const double what = s * (qhat - z);
                const double diff = w - what;
                acc[k - 1] = acc[k - 1] + diff * diff;
            }
        }
    }
    return true;
}

// Greedy binary-coded quantisation of one matrix; accumulates the residual per k.
bool encode_bcq_matrix(const Mat& m, int B, int G, uint32_t* mat_planes, uint16_t* mat_meta,
                       double* acc) {
    const int ng = m.C / G;
    const uint64_t plane_words = static_cast<uint64_t>(m.R) * m.C / 32;
    const uint64_t meta_plane = static_cast<uint64_t>(m.R) * ng;
    std::vector<double> res(G);
    std::vector<double> alpha(static_cast<size_t>(B) * ng);
    std::vector<unsigned> code(m.C);
    for (int r = 0; r < m.R; ++r) {
        const float* wr = m.w + static_cast<uint64_t>(r) * m.C;
        for (int g = 0; g < ng; ++g) {
            for (int j = 0; j < G; ++j) res[j] = wr[g * G + j];
            for (int j = 0; j < G; ++j) code[g * G + j] = 0;
            for (int i = 0; i < B; ++i) {
                double total = 0.0;
                for (int j = 0; j < G; ++j) total = total + std::fabs(res[j]);
                const uint16_t ab = f64_to_f16_bits(total / static_cast<double>(G));
                const double a = f16_bits_to_f64(ab);
                if (!std::isfinite(a)) return false;
                alpha[static_cast<size_t>(i) * ng + g] = a;
                mat_meta[static_cast<uint64_t>(i) * meta_plane + static_cast<uint64_t>(r) * ng + g] = ab;
                for (int j = 0; j < G; ++j) {
                    const bool pos = res[j] >= 0.0;
                    if (pos) code[g * G + j] |= 1u << (B - 1 - i);
                    res[j] = res[j] - a * (pos ? 1.0 : -1.0);
                }
            }
        }
        for (int c = 0; c < m.C; ++c) {
            set_code(mat_planes, plane_words, m.R, m.C, r, c, code[c], B, false);
            const double w = wr[c];
            for (int k = 1; k <= B; ++k) {
                double what = 0.0;
                for (int i = 0; i < k; ++i) {
                    const bool pos = (code[c] >> (B - 1 - i)) & 1u;
                    what = what + alpha[static_cast<size_t>(i) * ng + c / G] * (pos ? 1.0 : -1.0);
                }
                const double diff = w - what;
                acc[k - 1] = acc[k - 1] + diff * diff;
            }
        }
    }
    return true;
}

bool encode_one_expert(const EncodeJob& job, int local_e) {
    const dpa_layer_desc& d = *job.d;
    const int e = job.e_begin + local_e;
    const int H = d.hidden, I = d.inter, B = d.bits, G = d.group;
    const uint64_t gate_off = static_cast<uint64_t>(local_e) * I * H;
    const Mat mats[3] = {{job.wg + gate_off, I, H}, {job.wu + gate_off, I, H},
                         {job.wd + static_cast<uint64_t>(local_e) * H * I, H, I}};
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint8_t* ep = job.planes + static_cast<uint64_t>(e) * job.sz.planes_per_expert;
    uint8_t* em = job.meta + static_cast<uint64_t>(e) * job.sz.meta_per_expert;
    std::memset(ep, 0, job.sz.planes_per_expert);
    for (int m = 0; m < 3; ++m) {
        uint32_t* mp = reinterpret_cast<uint32_t*>(ep + job.sz.planes_matrix_offset[m]);
        uint16_t* mm = reinterpret_cast<uint16_t*>(em + job.sz.meta_matrix_offset[m]);
        const bool ok = d.format == DPA_FMT_UNIFORM ? encode_uniform_matrix(mats[m], B, G, mp, mm, acc)
                                                    : encode_bcq_matrix(mats[m], B, G, mp, mm, acc);
        if (!ok) return false;
    }
    for (int k = 0; k < B; ++k) job.rtable[static_cast<uint64_t>(e) * B + k] = acc[k];
    return true;
}

}  // namespace

extern "C" dpa_status dpa_encode(const dpa_layer_desc* desc, int e_begin, int n_e, const float* w_gate,
                                 const float* w_up, const float* w_down, void* planes, void* meta,
                                 double* rtable, int n_threads) {
    dpa_sizes sz;
    dpa_status st = dpa_encoded_sizes(desc, &sz);
    if (st != DPA_OK) return st;
    if (!w_gate || !w_up || !w_down || !planes || !meta || !rtable) return DPA_ERR_INVALID_ARG;
    if (e_begin < 0 || n_e < 0 || e_begin + n_e > desc->n_experts) return DPA_ERR_INVALID_ARG;
    if (n_e == 0) return DPA_OK;
    EncodeJob job{desc, sz, w_gate, w_up, w_down, static_cast<uint8_t*>(planes),
                  static_cast<uint8_t*>(meta), rtable, e_begin};
    unsigned hw = std::thread::hardware_concurrency();
    int nt = n_threads > 0 ? n_threads : static_cast<int>(hw ? hw : 1);
    nt = std::min(nt, n_e);
    std::atomic<int> next{0};
    std::atomic<bool> ok{true};
    auto worker = [&]() {
        for (;;) {
            const int i = next.fetch_add(1);
            if (i >= n_e) break;
            if (!encode_one_expert(job, i)) ok.store(false);
        }
    };
    if (nt <= 1) {
        worker();
    } else {
        std::vector<std::thread> th;
        th.reserve(nt);
        for (int t = 0; t < nt; ++t) th.emplace_back(worker);
        for (auto& t : th) t.join();
    }
    return ok.load() ? DPA_OK : DPA_ERR_INVALID_ARG;
}

namespace {

// Per input channel j of expert e: T[k-1][j] = sum over the rows of gate, then of up, of
// (w - w_k)^2 for the stored codes read at k planes (rows in order, one fp64 sum per channel).
bool distortion_one_expert(const dpa_layer_desc& d, const dpa_sizes& sz, int e, const float* wg, const float* wu,
                           const uint8_t* planes, const uint8_t* meta, double* T) {
    const int H = d.hidden, I = d.inter, B = d.bits, G = d.group, ng = H / G;
    const uint64_t plane_words = static_cast<uint64_t>(I) * H / 32;
    std::vector<double> acc(static_cast<size_t>(B) * H, 0.0);
    for (int m = 0; m < 2; ++m) {
        const float* w = m == 0 ? wg : wu;
        const uint32_t* mp = reinterpret_cast<const uint32_t*>(planes + static_cast<uint64_t>(e) * sz.planes_per_expert +
                                                               sz.planes_matrix_offset[m]);
        const uint16_t* mm = reinterpret_cast<const uint16_t*>(meta + static_cast<uint64_t>(e) * sz.meta_per_expert +
                                                               sz.meta_matrix_offset[m]);
        for (int r = 0; r < I; ++r) {
            for (int c = 0; c < H; ++c) {
                const unsigned code = get_code(mp, plane_words, H, r, c, B, d.format == DPA_FMT_UNIFORM);
                const double wv = w[static_cast<uint64_t>(r) * H + c];
                for (int k = 1; k <= B; ++k) {
                    double what;
                    if (d.format == DPA_FMT_UNIFORM) {
                        const double s = f16_bits_to_f64(mm[(static_cast<uint64_t>(r) * ng + c / G) * 2]);
                        const double z = f16_bits_to_f64(mm[(static_cast<uint64_t>(r) * ng + c / G) * 2 + 1]);
                        const int dsh = B - k;
                        const double qk = static_cast<double>(code >> dsh);
                        const double pw = static_cast<double>(1u << dsh);
                        what = s * ((qk * pw + (pw - 1.0) / 2.0) - z);
                    } else {
                        what = 0.0;
                        for (int i = 0; i < k; ++i) {
                            const double a = f16_bits_to_f64(
                                mm[static_cast<uint64_t>(i) * I * ng + static_cast<uint64_t>(r) * ng + c / G]);
                            what = what + a * (((code >> (B - 1 - i)) & 1u) ? 1.0 : -1.0);
                        }
                    }
                    const double diff = wv - what;
                    acc[static_cast<size_t>(k - 1) * H + c] = acc[static_cast<size_t>(k - 1) * H + c] + diff * diff;
                }
            }
        }
    }
    for (size_t i = 0; i < acc.size(); ++i) T[i] = acc[i];
    return true;
}

}  // namespace

extern "C" dpa_status dpa_distortion_tensor(const dpa_layer_desc* desc, int e_begin, int n_e, const float* w_gate,
                                            const float* w_up, const void* planes, const void* meta, double* T,
                                            int n_threads) {
    dpa_sizes sz;
    dpa_status st = dpa_encoded_sizes(desc, &sz);
    if (st != DPA_OK) return st;
    if (!w_gate || !w_up || !planes || !meta || !T) return DPA_ERR_INVALID_ARG;
    if (e_begin < 0 || n_e < 0 || e_begin + n_e > desc->n_experts) return DPA_ERR_INVALID_ARG;
    if (n_e == 0) return DPA_OK;
    const uint64_t per = static_cast<uint64_t>(desc->inter) * desc->hidden;
    const uint64_t tper = static_cast<uint64_t>(desc->bits) * desc->hidden;
    unsigned hw = std::thread::hardware_concurrency();
    int nt = n_threads > 0 ? n_threads : static_cast<int>(hw ? hw : 1);
    nt = std::min(nt, n_e);
    std::atomic<int> next{0};
    auto worker = [&]() {
        for (;;) {
            const int i = next.fetch_add(1);
            if (i >= n_e) break;
            const int e = e_begin + i;
            distortion_one_expert(*desc, sz, e, w_gate + i * per, w_up + i * per, static_cast<const uint8_t*>(planes),
                                  static_cast<const uint8_t*>(meta), T + static_cast<uint64_t>(e) * tper);
        }
    };
    if (nt <= 1) {
        worker();
    } else {
        std::vector<std::thread> th;
        th.reserve(nt);
        for (int t = 0; t < nt; ++t) th.emplace_back(worker);
        for (auto& t : th) t.join();
    }
    return DPA_OK;
}

extern "C" dpa_status dpa_export_codes(const dpa_layer_desc* desc, const void* planes, int expert,
                                       int matrix, uint8_t* codes) {
    dpa_sizes sz;
    dpa_status st = dpa_encoded_sizes(desc, &sz);
    if (st != DPA_OK) return st;
    if (!planes || !codes || expert < 0 || expert >= desc->n_experts || matrix < 0 || matrix > 2)
        return DPA_ERR_INVALID_ARG;
    const int R = matrix == DPA_MAT_DOWN ? desc->hidden : desc->inter;
    const int C = matrix == DPA_MAT_DOWN ? desc->inter : desc->hidden;
    const int B = desc->bits;
    const uint32_t* mp = reinterpret_cast<const uint32_t*>(
        static_cast<const uint8_t*>(planes) + static_cast<uint64_t>(expert) * sz.planes_per_expert +
        sz.planes_matrix_offset[matrix]);
    const uint64_t plane_words = static_cast<uint64_t>(R) * C / 32;
    for (int r = 0; r < R; ++r) {
        for (int c = 0; c < C; ++c) {
            codes[static_cast<uint64_t>(r) * C + c] =
                static_cast<uint8_t>(get_code(mp, plane_words, C, r, c, B, desc->format == DPA_FMT_UNIFORM));
        }
    }
    return DPA_OK;
}

extern "C" dpa_status dpa_export_meta(const dpa_layer_desc* desc, const void* meta, int expert, int matrix,
                                      float* s_or_alpha, float* zero) {
    dpa_sizes sz;
    dpa_status st = dpa_encoded_sizes(desc, &sz);
    if (st != DPA_OK) return st;
    if (!meta || !s_or_alpha || expert < 0 || expert >= desc->n_experts || matrix < 0 || matrix > 2)
        return DPA_ERR_INVALID_ARG;
    const int R = matrix == DPA_MAT_DOWN ? desc->hidden : desc->inter;
    const int C = matrix == DPA_MAT_DOWN ? desc->inter : desc->hidden;
    const int ng = C / desc->group;
    const uint16_t* mm = reinterpret_cast<const uint16_t*>(
        static_cast<const uint8_t*>(meta) + static_cast<uint64_t>(expert) * sz.meta_per_expert +
        sz.meta_matrix_offset[matrix]);
    if (desc->format == DPA_FMT_UNIFORM) {
        if (!zero) return DPA_ERR_INVALID_ARG;
        for (uint64_t i = 0; i < static_cast<uint64_t>(R) * ng; ++i) {
            s_or_alpha[i] = static_cast<float>(f16_bits_to_f64(mm[2 * i]));
            zero[i] = static_cast<float>(f16_bits_to_f64(mm[2 * i + 1]));
        }
    } else {
        for (uint64_t i = 0; i < static_cast<uint64_t>(desc->bits) * R * ng; ++i)
            s_or_alpha[i] = static_cast<float>(f16_bits_to_f64(mm[i]));
    }
    return DPA_OK;
}

// ---------------------------------------------------------------------------------------
// Per-expert stored widths (MatMoE, review "Core Contribution": an offline ILP over each
// expert's maximum bit-width under a memory budget). Exact dynamic programming over the experts
// from the last; every fp64 operation is a separate rounding (this file is built without
// contraction), so the result is reproducible by any IEEE implementation of the same steps.
// ---------------------------------------------------------------------------------------
extern "C" dpa_status dpa_solve_stored_widths(const dpa_layer_desc* desc, const double* importance,
                                              const double* rtable, int64_t budget_planes, uint8_t* widths) {
    dpa_sizes sz;
    const dpa_status st = dpa_encoded_sizes(desc, &sz);
    if (st != DPA_OK) return st;
    if (!importance || !rtable || !widths) return DPA_ERR_INVALID_ARG;
    const int E = desc->n_experts, B = desc->bits, kmin = desc->kmin, kmax = desc->kmax;
    for (int e = 0; e < E; ++e)
        if (!(importance[e] >= 0.0 && importance[e] <= 1.0e300)) return DPA_ERR_INVALID_ARG;
    if (budget_planes < static_cast<int64_t>(E) * kmin) return DPA_ERR_INVALID_ARG;
    const int64_t cap = static_cast<int64_t>(E) * kmax;
    const int U = static_cast<int>(budget_planes < cap ? budget_planes : cap);
    const double inf = std::numeric_limits<double>::infinity();
    std::vector<double> f(static_cast<size_t>(U) + 1, 0.0), g(static_cast<size_t>(U) + 1);
    std::vector<uint8_t> choice(static_cast<size_t>(E) * (U + 1), 0);
    for (int e = E - 1; e >= 0; --e) {
        const int need_after = kmin * (E - e - 1);
        for (int u = 0; u <= U; ++u) {
            double best = inf;
            int bb = 0;
            for (int b = kmin; b <= kmax; ++b) {
                if (u - b < need_after) break;
                const double t = importance[e] * rtable[static_cast<size_t>(e) * B + (b - 1)];
                const double v = t + f[u - b];
                if (v < best) {
                    best = v;
                    bb = b;
                }
            }
            g[u] = best;
            choice[static_cast<size_t>(e) * (U + 1) + u] = static_cast<uint8_t>(bb);
        }
        f.swap(g);
    }
    int u = U;
    for (int e = 0; e < E; ++e) {
        const int b = choice[static_cast<size_t>(e) * (U + 1) + u];
        widths[e] = static_cast<uint8_t>(b);
        u -= b;
    }
    return DPA_OK;
}

namespace {
// bytes of one plane of one matrix, and of one plane's (or, uniform, the matrix's) scale data
struct CompactGeom {
    uint64_t plane_bytes;    // R * C / 8 (the same for gate, up and down)
    uint64_t meta_matrix;    // uniform: a matrix's {s, z}; binary-coded: one plane's alphas
};
CompactGeom compact_geom(const dpa_layer_desc* d) {
    CompactGeom g;
    g.plane_bytes = static_cast<uint64_t>(d->hidden) * d->inter / 8;
    const uint64_t groups = static_cast<uint64_t>(d->inter) * (d->hidden / d->group);   // R * C/G per matrix
    g.meta_matrix = d->format == DPA_FMT_UNIFORM ? groups * 4 : groups * 2;
    return g;
}
bool widths_ok(const dpa_layer_desc* d, const uint8_t* widths) {
    for (int e = 0; e < d->n_experts; ++e)
        if (widths[e] < d->kmin || widths[e] > d->kmax) return false;
    return true;
}
uint64_t compact_expert_planes(const CompactGeom& g, int w) { return 3ull * w * g.plane_bytes; }
uint64_t compact_expert_meta(const dpa_layer_desc* d, const CompactGeom& g, int w) {
    return d->format == DPA_FMT_UNIFORM ? 3ull * g.meta_matrix : 3ull * w * g.meta_matrix;
}
}  // namespace

extern "C" dpa_status dpa_compact_sizes(const dpa_layer_desc* desc, const uint8_t* widths, uint64_t* planes_bytes,
                                        uint64_t* meta_bytes) {
    dpa_sizes sz;
    const dpa_status st = dpa_encoded_sizes(desc, &sz);
    if (st != DPA_OK) return st;
    if (!widths || !planes_bytes || !meta_bytes || !widths_ok(desc, widths)) return DPA_ERR_INVALID_ARG;
    const CompactGeom g = compact_geom(desc);
    uint64_t pb = 0, mb = 0;
    for (int e = 0; e < desc->n_experts; ++e) {
        pb += compact_expert_planes(g, widths[e]);
        mb += compact_expert_meta(desc, g, widths[e]);
    }
    *planes_bytes = pb;
    *meta_bytes = mb;
    return DPA_OK;
}

extern "C" dpa_status dpa_compact_layer(const dpa_layer_desc* desc, const void* planes, const void* meta,
                                        const uint8_t* widths, void* planes_out, void* meta_out, uint64_t* offsets) {
    dpa_sizes sz;
    const dpa_status st = dpa_encoded_sizes(desc, &sz);
    if (st != DPA_OK) return st;
    if (!planes || !meta || !widths || !planes_out || !meta_out || !offsets || !widths_ok(desc, widths))
        return DPA_ERR_INVALID_ARG;
    const CompactGeom g = compact_geom(desc);
    const uint8_t* pin = static_cast<const uint8_t*>(planes);
    const uint8_t* min_ = static_cast<const uint8_t*>(meta);
    uint8_t* pout = static_cast<uint8_t*>(planes_out);
    uint8_t* mout = static_cast<uint8_t*>(meta_out);
    uint64_t po = 0, mo = 0;
    for (int e = 0; e < desc->n_experts; ++e) {
        const int w = widths[e];
        offsets[2 * e] = po;
        offsets[2 * e + 1] = mo;
        for (int m = 0; m < 3; ++m) {   // the first w planes of each matrix: a prefix of its bytes
            const uint8_t* src = pin + static_cast<uint64_t>(e) * sz.planes_per_expert + sz.planes_matrix_offset[m];
            std::memcpy(pout + po, src, w * g.plane_bytes);
            po += w * g.plane_bytes;
        }
        for (int m = 0; m < 3; ++m) {
            const uint8_t* src = min_ + static_cast<uint64_t>(e) * sz.meta_per_expert + sz.meta_matrix_offset[m];
            const uint64_t n = desc->format == DPA_FMT_UNIFORM ? g.meta_matrix : w * g.meta_matrix;
            std::memcpy(mout + mo, src, n);
            mo += n;
        }
    }
    return DPA_OK;
}
