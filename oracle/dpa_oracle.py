"""Plain fp64 CPU oracle for the routed MoE expert FFN over prefix-decodable bitplane weights.

TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
benchmark's CPU-baseline leg may import or run this module. The product (the
CUDA library behind include/dpa.h) never calls it, and it shares no code with
that library: it is written from the pages, step by step, in the pages'
notation, with numpy/Python fp64 arithmetic and no blocking or fusion.

Pages (cited by title and section):
  [DPA]  DPA-MoE: A Runtime Precision Control Framework for MoE Inference, Abstract
         (prefix-decodable chunks, SharedScale AnyBCQ, offline per-expert residuals,
          post-routing allocation from live router gate scores, matched budgets)
  [DUO]  DuoRate: Two-Rate Per-Expert Precision Allocation for MoE Serving, Abstract
         (prefix-readable weight stream, distortion tensor, Lagrangian rate-distortion
          allocation solved by a bisection, prefill reads at the stored rate)
  [MAT]  MatMoE: Matryoshka Mixture-of-Experts with Dynamic Mixed-Precision Quantization,
         Abstract and review section "Core Contribution"
         (floor-and-compensation, bitplane storage, routing-score driven bit-widths
          found by a binary search to a target average bit-width, an offline ILP over each
          expert's maximum bit-width under a memory budget)

Where the pages leave a step open, the reading taken is stated at the function.

Parity status of each function (what pins it; see tests/test_oracle_pins.py):
  fp16_round          pinned: exact rational rounding on tie/near-tie values
  quantize_uniform    pinned: hand-worked group with exact values; range/error bounds
  fc_code / dequant   pinned: closed forms (k=B exact, zero-mean compensation, max error,
                      bit-pattern identity); planted no-compensation control fails
  encode (r table)    pinned: exact rational sum on small inputs; monotone in k;
                      ~4x per plane for uniform codes (closed-form approximation)
  encode_bcq_matrix   pinned: hand-worked group with exact signs, alphas, w_hat(k) and
  / dequant_bcq       residuals (tests/golden/bcq_worked_group.json); exact-rational greedy fit
                      and residual table on random experts; equal-magnitude closed form;
                      planted sign and plane-index mistakes fail the pin
  dexp                pinned: within 1 ulp of a correctly rounded exp (decimal module)
  route               pinned: logit = exact rational dot product rounded once; brute-force
                      top-k; expert permutation equivariance; softmax identities
  allocate            pinned: brute-force constrained optimum (Everett) on tiny inputs,
                      budget criterion, endpoint targets, monotone N along the bisection
  allocate_uniform    pinned: closed form (sum = floor(target*P), spread <= 1, integer targets)
  calibrate_threshold pinned: brute force over the cut points of the score distribution;
  / allocate_threshold endpoints; two plane counts and equal residuals reduce the Lagrangian
                      allocation of a batch to the threshold calibrated on that batch
  distortion_tensor   pinned: channel sums equal the gate+up residual (exact rational, small)
  prefill_profile     pinned: exact rational mean squares; counts by brute force
  tree_dot            pinned: within a few ulps of the exact rational dot product; order check
  solve_expert_rates  pinned: brute-force count-weighted optimum (Everett) on tiny inputs;
                      frequency cancels (scaling counts leaves every k(lambda) unchanged);
                      endpoint targets; monotone plane count along the bisection
  routing_mass        pinned: equals an independent scatter-add of the gates
  solve_stored_widths pinned: lexicographically smallest optimum by exhaustive enumeration
                      (exact integer data, non-convex residuals so greedy upgrades fail);
                      endpoint budgets (all kmin, all kmax); cost non-increasing in the budget
  allocate (cap)      pinned: k never above the width; width kmax for all = no cap; width kmin
                      for all = every pair at kmin; budget criterion kept
  expert_ffn / moe    pinned: hand-worked tiny layer; top-1 identity; linearity of the
                      gate-weighted combine; prefix property (low bits ignored); at
                      target = kmax = B the layer equals a torch fp32 computation (topk,
                      softmax, textbook dequantisation, matmul, silu) on the dense weights
  rmsnorm / stack     pinned: closed form on constant vectors; composition check
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# ---------------------------------------------------------------------------
# Rounding helpers (storage formats named by the pages: fp16 scale/zero, bf16 activations)
# ---------------------------------------------------------------------------


def fp16_round(x) -> np.ndarray:
    """Round fp64 values to the nearest fp16 value (ties to even), returned as fp64.

    numpy converts float64 -> float16 in one correctly rounded step (no fp32 detour).
    """
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Uniform asymmetric group quantisation with one scale/zero shared by every k
# [DPA] (one scale shared by every prefix); [MAT] Core Contribution: the low-bit prefix and
# the full code use the same quantisation parameters.
# Reading: plain round-to-nearest (the trained-parameter variant needs data).
# ---------------------------------------------------------------------------


def quantize_uniform(w: np.ndarray, B: int, G: int):
    """Asymmetric B-bit codes per group of G consecutive inputs of each row.

    For each group: lo = min w, hi = max w (fp64);
      s = fp16(( hi - lo ) / (2^B - 1)), s := 1 if it rounds to 0;
      z = clamp(rint(-lo / s), 0, 2^B - 1);
      q = clamp(rint(w / s) + z, 0, 2^B - 1).
    rint rounds half to even. Returns q uint8 [R][C], s fp64 [R][C/G], z fp64 [R][C/G].
    """
    R, C = w.shape
    if C % G:
        raise ValueError("columns must be a multiple of the group size")
    qmax = float(2 ** B - 1)
    wg = np.asarray(w, dtype=np.float64).reshape(R, C // G, G)
    lo = wg.min(axis=-1)
    hi = wg.max(axis=-1)
    s = fp16_round((hi - lo) / qmax)
    s = np.where(s == 0.0, 1.0, s)
    if not np.all(np.isfinite(s)):
        raise ValueError("group range too large for an fp16 scale")
    z = np.clip(np.rint(-lo / s), 0.0, qmax)
    q = np.clip(np.rint(wg / s[..., None]) + z[..., None], 0.0, qmax)
    return q.reshape(R, C).astype(np.uint8), s, z


def fc_code(q, B: int, k: int) -> np.ndarray:
    """Floor-and-compensation code [MAT] Core Contribution (F&C) and Abstract item (2).

    Keep the k most significant of the B code bits (floor to a multiple of 2^(B-k))
    and add the mean of the dropped, uniformly distributed residual, (2^(B-k) - 1)/2:
        q_hat = (q >> (B-k)) * 2^(B-k) + (2^(B-k) - 1) / 2
    """
    if not 1 <= k <= B:
        raise ValueError("k out of range")
    d = B - k
    qk = np.right_shift(np.asarray(q, dtype=np.int64), d)
    return qk.astype(np.float64) * float(2 ** d) + (float(2 ** d) - 1.0) / 2.0


def dequant_uniform(q, s, z, B: int, k: int, G: int) -> np.ndarray:
    """w_hat = s * (q_hat - z), with s, z broadcast over each group of G inputs."""
    qh = fc_code(q, B, k)
    R, C = qh.shape
    sg = np.repeat(np.asarray(s, np.float64), G, axis=1)
    zg = np.repeat(np.asarray(z, np.float64), G, axis=1)
    return sg * (qh - zg)


def bitplanes(q, B: int) -> np.ndarray:
    """MSB-first bitplanes [MAT] Core Contribution (bitplane storage): plane p holds bit (B-1-p)."""
    q = np.asarray(q, dtype=np.int64)
    return np.stack([(q >> (B - 1 - p)) & 1 for p in range(B)]).astype(np.uint8)


def codes_from_planes(planes, k: int, B: int) -> np.ndarray:
    """Truncated code from the first k planes only: sum_{p<k} plane_p * 2^(B-1-p)."""
    out = np.zeros(planes.shape[1:], dtype=np.int64)
    for p in range(k):
        out += planes[p].astype(np.int64) << (B - 1 - p)
    return out


# ---------------------------------------------------------------------------
# Binary-coded quantisation, greedy fit ([DPA] "AnyBCQ"): W ~ sum_{i<k} alpha_i * b_i
# Reading: each group of G inputs has its own fp16 alpha_i; signs chosen greedily on
# the running residual, sign(0) = +1; alpha_i is the least-squares scale for those
# signs, mean |R| over the group, summed in input order.
# ---------------------------------------------------------------------------


def encode_bcq_matrix(w: np.ndarray, B: int, G: int):
    """Returns signs bool [B][R][C] (True <-> +1) and alpha fp64 [B][R][C/G] (fp16 values)."""
    R, C = w.shape
    res = np.asarray(w, dtype=np.float64).reshape(R, C // G, G).copy()
    signs = np.empty((B, R, C // G, G), dtype=bool)
    alpha = np.empty((B, R, C // G), dtype=np.float64)
    for i in range(B):
        pos = res >= 0.0
        b = np.where(pos, 1.0, -1.0)
        total = np.cumsum(np.abs(res), axis=-1)[..., -1]   # sequential sum in input order
        a = fp16_round(total / float(G))
        res = res - a[..., None] * b
        signs[i] = pos
        alpha[i] = a
    return signs.reshape(B, R, C), alpha


def dequant_bcq(signs, alpha, k: int, G: int) -> np.ndarray:
    """w_hat^(k) = sum_{i<k} alpha_i * b_i, summed in plane order."""
    B, R, C = signs.shape
    out = np.zeros((R, C), dtype=np.float64)
    for i in range(k):
        b = np.where(signs[i], 1.0, -1.0)
        out = out + np.repeat(alpha[i], G, axis=1) * b
    return out


# ---------------------------------------------------------------------------
# Offline per-expert residual table ([DPA] "profiles per-expert reconstruction residuals
# offline"; [DUO] "bakes a distortion tensor").
# Reading: r_e(k) = ||W_e - W_hat_e^(k)||_F^2 over gate, up and down together, for k = 1..B,
# accumulated as one sequential fp64 sum in the order gate rows, up rows, down rows.
# ---------------------------------------------------------------------------


def _sequential_sum_of_squares(diffs: Sequence[np.ndarray]) -> float:
    flat = np.concatenate([np.asarray(d, np.float64).ravel() for d in diffs])
    sq = flat * flat
    return float(np.cumsum(sq)[-1]) if sq.size else 0.0


def encode_expert(gate: np.ndarray, up: np.ndarray, down: np.ndarray, fmt: int, B: int, G: int):
    """Encode one expert's three matrices and compute r[k-1] = r_e(k), k = 1..B.

    fmt 0 (uniform): returns {"q": [q_g, q_u, q_d], "s": [...], "z": [...], "r": r}
    fmt 1 (BCQ):     returns {"signs": [...], "alpha": [...], "r": r}
    """
    mats = (gate, up, down)
    r = np.zeros(B, dtype=np.float64)
    if fmt == 0:
        enc = [quantize_uniform(m, B, G) for m in mats]
        for k in range(1, B + 1):
            diffs = [m.astype(np.float64) - dequant_uniform(q, s, z, B, k, G)
                     for m, (q, s, z) in zip(mats, enc)]
            r[k - 1] = _sequential_sum_of_squares(diffs)
        return {"q": [e[0] for e in enc], "s": [e[1] for e in enc], "z": [e[2] for e in enc], "r": r}
    enc = [encode_bcq_matrix(m, B, G) for m in mats]
    for k in range(1, B + 1):
        diffs = [m.astype(np.float64) - dequant_bcq(sg, al, k, G) for m, (sg, al) in zip(mats, enc)]
        r[k - 1] = _sequential_sum_of_squares(diffs)
    return {"signs": [e[0] for e in enc], "alpha": [e[1] for e in enc], "r": r}


def dequant_expert(enc: Dict, fmt: int, B: int, k: int, G: int) -> List[np.ndarray]:
    """Dense fp64 (gate, up, down) of an encoded expert read at k planes."""
    if fmt == 0:
        return [dequant_uniform(q, s, z, B, k, G) for q, s, z in zip(enc["q"], enc["s"], enc["z"])]
    return [dequant_bcq(sg, al, k, G) for sg, al in zip(enc["signs"], enc["alpha"])]


# ---------------------------------------------------------------------------
# exp for the router softmax.
# Reading: the pages fix no exp; routing must be reproducible bit for bit, so both sides
# evaluate one fixed fp64 procedure: Cody & Waite (1980) argument reduction with ln 2 split
# in two parts, a degree-13 Taylor polynomial in Horner form, then scaling by 2^n. Every
# operation is one IEEE round-to-nearest fp64 operation (Python floats do exactly that).
# Results below the fp64 normal range (x < -708) are returned as 0.
# ---------------------------------------------------------------------------

# 1/ln 2 rounded to nearest; ln 2 cut after 42 fractional bits (so n * LN2_HI is exact for
# |n| < 2^11), and the rounded remainder. Derived with the decimal module from ln 2.
INV_LN2 = float.fromhex("0x1.71547652b82fep+0")
LN2_HI = float.fromhex("0x1.62e42fefa3800p-1")
LN2_LO = float.fromhex("0x1.ef35793c76730p-45")
# 1/i! rounded to nearest, i = 0..13
EXP_TAYLOR = tuple(float(Fraction(1, math.factorial(i))) for i in range(14))
EXP_FLUSH_BELOW = -708.0


def dexp(x: float) -> float:
    x = float(x)
    if x < EXP_FLUSH_BELOW:
        return 0.0
    n = round(x * INV_LN2)           # Python round(): half to even
    nf = float(n)
    r = (x - nf * LN2_HI) - nf * LN2_LO
    p = EXP_TAYLOR[13]
    for i in range(12, -1, -1):
        p = p * r + EXP_TAYLOR[i]    # two roundings: Python does not fuse
    return math.ldexp(p, n)


# ---------------------------------------------------------------------------
# Router: softmax top-k gating ([DPA] "routing each token to a small set of experts").
# Readings: logit l[t][e] = the exact dot product of the bf16 token and router row, rounded
# once to fp64 (bf16 x bf16 products are exact in fp64; math.fsum returns the correctly
# rounded sum). Top-k by descending logit, ties to the lower expert id. Gates:
#   norm_topk = 1: g_i = exp(l_i - l_max) / sum over the k selected (slot order);
#   norm_topk = 0: g_i = exp(l_i - l_max) / sum over all experts (ascending expert id).
# ---------------------------------------------------------------------------


def router_logits(x_bits: np.ndarray, wr_bits: np.ndarray) -> np.ndarray:
    x = bf16_bits_to_f64(x_bits)
    w = bf16_bits_to_f64(wr_bits)
    T, E = x.shape[0], w.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    for t in range(T):
        prods = x[t][None, :] * w            # exact
        for e in range(E):
            out[t, e] = math.fsum(prods[e].tolist())
    return out


def topk_select(logits_row: np.ndarray, K: int) -> List[int]:
    order = sorted(range(len(logits_row)), key=lambda e: (-float(logits_row[e]), e))
    return order[:K]


def gates_from_logits(logits_row: np.ndarray, sel: Sequence[int], norm_topk: int) -> List[float]:
    lmax = float(logits_row[sel[0]])
    num = [dexp(float(logits_row[e]) - lmax) for e in sel]
    den = 0.0
    if norm_topk:
        for v in num:
            den = den + v
    else:
        for e in range(len(logits_row)):
            den = den + dexp(float(logits_row[e]) - lmax)
    return [v / den for v in num]


def route(x_bits: np.ndarray, wr_bits: np.ndarray, K: int, norm_topk: int,
          logits: Optional[np.ndarray] = None):
    """Returns (idx int32 [T][K], gates fp64 [T][K], logits fp64 [T][E])."""
    if logits is None:
        logits = router_logits(x_bits, wr_bits)
    T = logits.shape[0]
    idx = np.empty((T, K), dtype=np.int32)
    g = np.empty((T, K), dtype=np.float64)
    for t in range(T):
        sel = topk_select(logits[t], K)
        idx[t] = sel
        g[t] = gates_from_logits(logits[t], sel, norm_topk)
    return idx, g, logits


# ---------------------------------------------------------------------------
# Post-routing plane allocation ([DPA] "allocates chunks at inference time using live router
# gate scores"; [DUO] "Lagrangian rate-distortion allocation ... a bisection";
# [MAT] "binary search ... to hit a target average bit-width").
# Readings: one multiplier lambda per call (per layer and batch). Each routed pair p
# (token t, slot j, expert e, gate g) picks
#     k_p(lambda) = argmin_{kmin <= k <= kmax} fl( fl(g * r_e(k)) + fl(lambda * k) ),
# ties to the smaller k. N(lambda) = sum_p k_p(lambda). The budget is target * P planes
# (target = average planes per routed pair). Bisection, exactly 64 steps:
#     lo = 0, hi = 2 * max_p fl(g_p * r_e(kmin)) + 1
#     mid = 0.5 * (lo + hi); if N(mid) > budget: lo = mid else hi = mid
# and the answer is lambda = hi, k = k(hi), so the average never exceeds the target.
# ---------------------------------------------------------------------------


def pair_costs(idx: np.ndarray, gates: np.ndarray, r: np.ndarray, kmin: int, kmax: int,
               cap: Optional[np.ndarray] = None) -> np.ndarray:
    """c[p][k - kmin] = fl(g_p * r_{e_p}(k)) for the pairs in token-major, slot order; with
    per-expert stored widths `cap`, plane counts above the expert's width cost +inf (never
    chosen: an expert stored at b planes can be read at no more than b)."""
    e = idx.reshape(-1)
    g = gates.reshape(-1)
    ks = np.arange(kmin, kmax + 1)
    c = g[:, None] * r[e][:, ks - 1]
    if cap is not None:
        c = np.where(ks[None, :] > np.asarray(cap)[e][:, None], np.inf, c)
    return c


def choose_k(c: np.ndarray, lam: float, kmin: int, kmax: int) -> np.ndarray:
    ks = np.arange(kmin, kmax + 1, dtype=np.float64)
    cost = c + lam * ks[None, :]        # two separate roundings (numpy does not fuse)
    return (np.argmin(cost, axis=1) + kmin).astype(np.int64)   # argmin: first minimum


def allocate(idx: np.ndarray, gates: np.ndarray, r: np.ndarray, kmin: int, kmax: int,
             target: float, iters: int = 64, trace: Optional[list] = None, cap: Optional[np.ndarray] = None):
    """Returns (k int [T][K], lambda). `cap`: per-expert stored widths (k <= cap[e])."""
    if not (kmin <= target <= kmax):
        raise ValueError("target outside [kmin, kmax]")
    c = pair_costs(idx, gates, r, kmin, kmax, cap)
    P = c.shape[0]
    budget = float(target) * float(P)
    lo = 0.0
    hi = 2.0 * float(np.max(c[:, 0])) + 1.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        n = int(choose_k(c, mid, kmin, kmax).sum())
        if trace is not None:
            trace.append((mid, n))
        if float(n) > budget:
            lo = mid
        else:
            hi = mid
    k = choose_k(c, hi, kmin, kmax)
    return k.reshape(idx.shape), hi


# ---------------------------------------------------------------------------
# Allocation policies other than the Lagrangian (the controls and the prior design the pages
# compare with).
# [DPA] Abstract: DPA-MoE is compared with "uniform chunk allocation at matched budgets".
#   Reading: every routed pair gets an equal share of the same plane budget floor(target * P)
#   (the Lagrangian's budget rule): k = floor(N / P) planes, and the first N mod P pairs in
#   token-major slot order one plane more. It ignores the gates.
# [MAT] Core Contribution: at run time an expert whose routing score is above a threshold runs
#   at high precision and the others at low precision; the threshold comes from a binary search
#   over a calibration distribution of routing scores so that the average bit-width meets the
#   target. Readings: the routing score is the pair's gate g; high = kmax, low = kmin planes; the
#   calibration distribution is the gates of a calibration batch's routed pairs; the search is
#   64 fp64 bisection steps on [0, 1] (gates lie in [0, 1]) with the count of scores strictly
#   above the midpoint:
#       mid = 0.5 * (lo + hi); if kmin * n + (kmax - kmin) * #{s > mid} > target * n: lo = mid
#       else hi = mid,
#   and the threshold is hi, so the calibration average never exceeds the target. At run time
#   k = kmax if g > threshold else kmin, with no budget enforced on the live batch (the threshold
#   is fixed ahead of time).
# ---------------------------------------------------------------------------


def allocate_uniform(P: int, kmin: int, kmax: int, target: float) -> np.ndarray:
    """Equal shares of the budget floor(target * P) planes over the P pairs (token-major order)."""
    if not (kmin <= target <= kmax):
        raise ValueError("target outside [kmin, kmax]")
    n = int(math.floor(float(target) * float(P)))
    base, rem = divmod(n, P)
    return np.array([base + (1 if p < rem else 0) for p in range(P)], dtype=np.int64)


def calibrate_threshold(scores: np.ndarray, kmin: int, kmax: int, target: float, iters: int = 64,
                        trace: Optional[list] = None) -> float:
    """Threshold on the routing score so that the calibration scores' average plane count
    (kmax above the threshold, kmin otherwise) does not exceed the target."""
    if not (kmin <= target <= kmax):
        raise ValueError("target outside [kmin, kmax]")
    s = np.asarray(scores, dtype=np.float64).reshape(-1)
    n = s.size
    budget = float(target) * float(n)
    lo, hi = 0.0, 1.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        planes = kmin * n + (kmax - kmin) * int(np.count_nonzero(s > mid))
        if trace is not None:
            trace.append((mid, planes))
        if float(planes) > budget:
            lo = mid
        else:
            hi = mid
    return hi


def allocate_threshold(gates: np.ndarray, threshold: float, kmin: int, kmax: int) -> np.ndarray:
    """k = kmax where the pair's gate is above the threshold, else kmin."""
    g = np.asarray(gates, dtype=np.float64)
    return np.where(g > float(threshold), kmax, kmin).astype(np.int64)


# ---------------------------------------------------------------------------
# Workload-profiled per-expert read rates ([DUO] Abstract: one uniform tier of a prefix-readable
# stream is stored with a baked distortion tensor; online, the workload's own prefill is profiled
# without labels and a Lagrangian rate-distortion allocation is solved under the decode
# functional; routing frequency cancels from every per-expert decision; the solve is one dot
# product per expert and a bisection; prefill reads at the stored rate, decode at the workload's).
# Readings:
#   distortion tensor  T[e][k-1][j] = sum over the rows i of the gate and up projections of
#                      (W - W_hat^(k))[i][j]^2: the squared reconstruction error that input
#                      channel j meets at k planes (the down projection's input is internal to
#                      the expert and is not profiled);
#   profile            m[j] = (sum over the prefill tokens, in token order, of x[t][j]^2) / T and
#                      c[e] = the number of prefill pairs routed to expert e;
#   distortion         D_e(k) = <m, T[e][k-1]>, summed as 32 chunks of H/32 consecutive channels
#                      (each sequential from 0) combined by the pairwise tree
#                      p[i] + p[i+16], then + [i+8], + [i+4], + [i+2], + [i+1];
#   decode functional  expected planes read per selected expert: sum_e c_e k_e / sum_e c_e;
#   decision           k_e(lambda) = argmin_k fl(D_e(k) + fl(lambda * k)), ties to the smaller k:
#                      the objective sum_e c_e (D_e(k_e) + lambda k_e) separates per expert and
#                      c_e > 0 drops out of each argmin;
#   bisection          64 steps on [0, 2 max_e D_e(kmin) + 1]: if sum_e c_e k_e(mid) >
#                      target * sum_e c_e then lo = mid else hi = mid; lambda = hi. Experts the
#                      prefill never routed to get k_e(hi) too (they may be selected in decode).
# In decode every pair routed to e then reads k_e planes (the expert-rate table).
# ---------------------------------------------------------------------------


def distortion_tensor(enc: Dict, fmt: int, B: int, G: int, gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """T [B][H]: per input channel, the squared error of gate and up at k = 1..B planes."""
    H = gate.shape[1]
    out = np.zeros((B, H), dtype=np.float64)
    for k in range(1, B + 1):
        wg, wu, _ = dequant_expert(enc, fmt, B, k, G)
        dg = gate.astype(np.float64) - wg
        du = up.astype(np.float64) - wu
        for j in range(H):   # rows in order, gate then up, one sequential sum per channel
            col = np.concatenate([dg[:, j], du[:, j]])
            out[k - 1, j] = float(np.cumsum(col * col)[-1])
    return out


def prefill_profile(x_bits: np.ndarray, idx: np.ndarray, n_experts: int):
    """m [H] (mean square of each input channel over the prefill tokens) and c [E] (pair counts)."""
    x = bf16_bits_to_f64(x_bits)
    T, H = x.shape
    m = np.empty(H, dtype=np.float64)
    for j in range(H):
        acc = 0.0
        for t in range(T):
            acc = acc + x[t, j] * x[t, j]
        m[j] = acc / float(T)
    c = np.bincount(np.asarray(idx).reshape(-1), minlength=n_experts).astype(np.int64)
    return m, c


def tree_dot(m: np.ndarray, t: np.ndarray) -> float:
    """<m, t> in the fixed order above: 32 sequential chunk sums, then the pairwise tree."""
    H = m.size
    step = H // 32
    part = []
    for c in range(32):
        acc = 0.0
        for j in range(c * step, (c + 1) * step):
            acc = acc + float(m[j]) * float(t[j])
        part.append(acc)
    width = 16
    while width >= 1:
        part = [part[i] + part[i + width] for i in range(width)]
        width //= 2
    return part[0]


def solve_expert_rates(Tdist: np.ndarray, m: np.ndarray, counts: np.ndarray, kmin: int, kmax: int,
                       target: float, iters: int = 64):
    """k_e for every expert (int [E]) and lambda. Tdist: [E][B][H]."""
    if not (kmin <= target <= kmax):
        raise ValueError("target outside [kmin, kmax]")
    E = Tdist.shape[0]
    D = np.array([[tree_dot(m, Tdist[e, k - 1]) for k in range(kmin, kmax + 1)] for e in range(E)])
    ks = np.arange(kmin, kmax + 1, dtype=np.float64)

    def decide(lam):
        return (np.argmin(D + lam * ks[None, :], axis=1) + kmin).astype(np.int64)

    budget = float(target) * float(int(np.sum(counts)))
    lo, hi = 0.0, 2.0 * float(np.max(D[:, 0])) + 1.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        n = int(np.sum(np.asarray(counts, dtype=np.int64) * decide(mid)))
        if float(n) > budget:
            lo = mid
        else:
            hi = mid
    return decide(hi), hi, D


def allocate_expert_table(idx: np.ndarray, k_table: np.ndarray) -> np.ndarray:
    """Every pair reads its expert's rate."""
    return np.asarray(k_table, dtype=np.int64)[np.asarray(idx)]


# ---------------------------------------------------------------------------
# Expert FFN (SwiGLU) and gate-weighted combine.
#   a = W_gate^(k) x, u = W_up^(k) x, h = silu(a) * u, o = W_down^(k) h,
#   y_t = sum_{slots j} g_{t,j} o_{t,j}  (+ sum of shared experts, dense, gate 1).
# Reading: shared experts are dense bf16 and are neither allocated nor counted in the budget.
# ---------------------------------------------------------------------------


def silu(a):
    a = np.asarray(a, dtype=np.float64)
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def expert_ffn(x: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    a = wg @ x
    u = wu @ x
    h = silu(a) * u
    return wd @ h


def combine_token(gates_row: Sequence[float], outs: Sequence[np.ndarray],
                  shared_outs: Sequence[np.ndarray] = ()) -> np.ndarray:
    """y_t = sum over slots j, in slot order, of g_{t,j} * o_{t,j}, then + each shared expert's
    output (gate weight 1), accumulated in fp64 from zero."""
    acc = np.zeros(np.asarray(outs[0] if len(outs) else shared_outs[0]).shape)
    for g, o in zip(gates_row, outs):
        acc = acc + float(g) * o
    for o in shared_outs:
        acc = acc + o
    return acc


def shared_outputs(x_row: np.ndarray, shared) -> List[np.ndarray]:
    """Outputs of the always-on experts (dense bf16 weights) for one token."""
    if shared is None:
        return []
    sg, su, sd = shared
    return [expert_ffn(x_row, bf16_bits_to_f64(sg[s]), bf16_bits_to_f64(su[s]), bf16_bits_to_f64(sd[s]))
            for s in range(sg.shape[0])]


# ---------------------------------------------------------------------------
# Per-expert stored width ([MAT] Core Contribution: offline, an ILP picks each expert's maximum
# bit-width, 2/3/4, under a memory budget; the metric is routing score x Fisher-approximated
# Hessian x quantization error).
#   Readings: the routing score of expert e is its routing mass, the sum of the gates of its
#   routed pairs over a calibration batch (in token-major slot order); no Fisher information is
#   available, so the Hessian factor is 1; the quantization error at b stored planes is the
#   residual r_e(b). Every plane of every expert has the same size, so the memory budget is a
#   number of stored planes. The ILP
#       minimise sum_e fl(imp_e * r_e(b_e))  s.t.  sum_e b_e <= budget,  kmin <= b_e <= kmax
#   is solved exactly by dynamic programming over the experts from the last:
#       f(E, u) = 0;  f(e, u) = min_b fl(fl(imp_e * r_e(b)) + f(e+1, u - b)),
#   b over [kmin, kmax] with u - b >= kmin * (E - e - 1), ties to the smaller b; the widths
#   are read off from u = budget (clipped to E * kmax) forwards.
# ---------------------------------------------------------------------------


def routing_mass(idx: np.ndarray, gates: np.ndarray, n_experts: int) -> np.ndarray:
    """Sum of each expert's gates over the routed pairs, in token-major slot order."""
    m = np.zeros(n_experts, dtype=np.float64)
    for e, g in zip(idx.reshape(-1).tolist(), gates.reshape(-1).tolist()):
        m[e] = m[e] + g
    return m


def solve_stored_widths(importance: np.ndarray, r: np.ndarray, kmin: int, kmax: int, budget: int) -> np.ndarray:
    """Stored planes per expert (int [E]) minimising the importance-weighted residual."""
    E = len(importance)
    if budget < E * kmin:
        raise ValueError("budget below every expert at kmin")
    budget = min(int(budget), E * kmax)
    inf = float("inf")
    f = [0.0] * (budget + 1)                      # f(E, u)
    choice = [[0] * (budget + 1) for _ in range(E)]
    for e in range(E - 1, -1, -1):
        need_after = kmin * (E - e - 1)
        g = [inf] * (budget + 1)
        for u in range(budget + 1):
            best, bb = inf, 0
            for b in range(kmin, kmax + 1):
                if u - b < need_after:
                    break
                v = float(np.float64(importance[e]) * np.float64(r[e][b - 1])) + f[u - b]
                if v < best:
                    best, bb = v, b
            g[u], choice[e][u] = best, bb
        f = g
    widths, u = [], budget
    for e in range(E):
        b = choice[e][u]
        widths.append(b)
        u -= b
    return np.array(widths, dtype=np.int64)


ALLOC_LAGRANGE, ALLOC_UNIFORM, ALLOC_THRESHOLD, ALLOC_EXPERT_TABLE = 0, 1, 2, 3


def allocate_policy(policy: int, idx: np.ndarray, gates: np.ndarray, r_table: Optional[np.ndarray], kmin: int,
                    kmax: int, target: float, threshold: Optional[float] = None,
                    expert_k: Optional[np.ndarray] = None, cap: Optional[np.ndarray] = None):
    """Plane counts [T][K] and the policy's multiplier (lambda; the threshold; 0 for uniform and
    for the expert-rate table). With per-expert stored widths `cap`, the Lagrangian optimises
    within them (costs above a width are +inf) and the other policies' counts are clipped to
    them."""
    if policy == ALLOC_LAGRANGE:
        return allocate(idx, gates, r_table, kmin, kmax, target, cap=cap)
    if policy == ALLOC_EXPERT_TABLE:
        k, lam = allocate_expert_table(idx, expert_k), 0.0
    elif policy == ALLOC_UNIFORM:
        k, lam = allocate_uniform(idx.size, kmin, kmax, target).reshape(idx.shape), 0.0
    elif policy == ALLOC_THRESHOLD:
        k, lam = allocate_threshold(gates, threshold, kmin, kmax).reshape(idx.shape), float(threshold)
    else:
        raise ValueError("unknown allocation policy")
    if cap is not None:
        k = np.minimum(k, np.asarray(cap, dtype=np.int64)[idx])
    return k, lam


def moe_forward(x_bits: np.ndarray, wr_bits: np.ndarray, experts: Dict[int, Dict], shape,
                target: float, shared: Optional[Tuple[np.ndarray, np.ndarray, np.ndarray]] = None,
                r_table: Optional[np.ndarray] = None, logits: Optional[np.ndarray] = None,
                token_subset: Optional[Sequence[int]] = None, policy: int = ALLOC_LAGRANGE,
                threshold: Optional[float] = None, expert_k: Optional[np.ndarray] = None,
                widths: Optional[np.ndarray] = None):
    """One MoE layer. `experts` maps expert id -> encode_expert() output (only the experts that
    are routed to are needed); `r_table` is [E][B] (all experts' residuals; defaults to the
    encoded ones, which then must cover every expert). Returns y fp64 [T][H] (rows outside
    token_subset are NaN) and the decision-path results."""
    fmt, B, G = shape.fmt, shape.bits, shape.group
    idx, g, logits = route(x_bits, wr_bits, shape.top_k, shape.norm_topk, logits)
    if r_table is None and policy == ALLOC_LAGRANGE:
        r_table = np.stack([experts[e]["r"] for e in range(shape.n_experts)])
    k, lam = allocate_policy(policy, idx, g, r_table, shape.kmin, shape.kmax, target, threshold, expert_k,
                             cap=widths)
    x = bf16_bits_to_f64(x_bits)
    T = x.shape[0]
    toks = range(T) if token_subset is None else token_subset
    y = np.full((T, shape.hidden), np.nan)
    dense_cache: Dict[Tuple[int, int], List[np.ndarray]] = {}
    for t in toks:
        outs = []
        for j in range(shape.top_k):
            e, kk = int(idx[t, j]), int(k[t, j])
            if (e, kk) not in dense_cache:
                dense_cache[(e, kk)] = dequant_expert(experts[e], fmt, B, kk, G)
            wg, wu, wd = dense_cache[(e, kk)]
            outs.append(expert_ffn(x[t], wg, wu, wd))
        y[t] = combine_token(g[t], outs, shared_outputs(x[t], shared))
    return y, {"idx": idx, "gates": g, "logits": logits, "k": k, "lambda": lam}


# ---------------------------------------------------------------------------
# Stack glue between layers (pre-norm residual; the pages give no form, plainest reading):
#   h_{l+1} = h_l + MoE_l( bf16( RMSNorm(h_l) ) ),  RMSNorm(v) = v / sqrt(mean(v^2) + 1e-6)
# ---------------------------------------------------------------------------

RMS_EPS = 1e-6


def rmsnorm(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + RMS_EPS)


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp64 to bf16 (nearest, ties to even) in one step, via exact integer arithmetic."""
    a = np.asarray(a, dtype=np.float64)
    m, ex = np.frexp(a)                        # a = m * 2^ex, 0.5 <= |m| < 1
    sig = np.rint(np.ldexp(m, 8))              # 8 significant bits, ties to even
    out = np.ldexp(sig, ex - 8).astype(np.float32)   # exact: 8-bit significand
    return (out.view(np.uint32) >> 16).astype(np.uint16)
