"""Pins for the fp64 oracle: each check ties it to something other than itself
(hand-worked exact values, closed forms, exact rational arithmetic, brute force,
a correctly rounded exp), chosen so that a dropped term, a wrong sign or index or
a transposed operand in the oracle fails at least one of them. CPU only.
"""
import itertools
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

from oracle import dpa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers (exact arithmetic)

def rne_to_format(v: Fraction, mant_bits: int, emin: int) -> Fraction:
    """Round a rational to the nearest value of a binary format with `mant_bits` stored
    significand bits and minimum normal exponent `emin` (ties to even), no overflow."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - mant_bits)
    n = a / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def f64_ulp(x: float) -> float:
    return math.ulp(x)


# ----------------------------------------------------------------- fp16 rounding

def test_fp16_round_matches_exact_rounding_on_ties_and_near_ties():
    vals = [1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 1.0 + 2.0 ** -11 + 2.0 ** -40,
            1.0 + 2.0 ** -11 - 2.0 ** -40, 2.0 ** -24 * 1.5, 2.0 ** -24 * 2.5,
            0.1, 1.0 / 3.0, 1.875 / 15.0, 0.11666666666666667, 6.1e-5, 65504.0, -0.3 / 15]
    got = O.fp16_round(np.array(vals))
    for v, g in zip(vals, got):
        want = rne_to_format(Fraction(v), 10, -14)
        assert Fraction(float(g)) == want, (v, g, float(want))


# ----------------------------------------------------------------- uniform quantiser + F&C

def test_hand_worked_group_exact():
    fx = json.load(open(os.path.join(GOLDEN, "fc_worked_group.json")))
    B, G = fx["B"], fx["G"]
    w = np.array(fx["w"], dtype=np.float32)[None, :]
    q, s, z = O.quantize_uniform(w, B, G)
    assert float(s[0, 0]) == fx["s"] and float(z[0, 0]) == fx["z"]
    assert q[0].tolist() == fx["q"]
    for k in range(1, B + 1):
        wh = O.dequant_uniform(q, s, z, B, k, G)[0]
        assert wh.tolist() == fx["w_hat"][str(k)], k


def test_quantizer_clamps_and_scale_from_exact_rounding():
    # all-positive group: z would be negative and clamps to 0; the top code clamps to 15
    w = np.array([[0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0]], dtype=np.float32)
    q, s, z = O.quantize_uniform(w, 4, 8)
    s_exact = rne_to_format((Fraction(2.0) - Fraction(0.25)) / 15, 10, -14)
    assert Fraction(float(s[0, 0])) == s_exact
    assert z[0, 0] == 0.0
    sf = float(s_exact)
    want = [min(15, max(0, int(round(float(v) / sf)))) for v in w[0]]
    assert q[0].tolist() == want and q[0, -1] == 15


def test_quantizer_error_bound_random():
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    B, G = 4, 64
    q, s, z = O.quantize_uniform(w, B, G)
    assert q.min() >= 0 and q.max() <= 15
    wh = O.dequant_uniform(q, s, z, B, B, G)
    err = np.abs(w.astype(np.float64) - wh)
    # inside [lo, hi] the rounding error is at most s/2 plus the clamp of one rounding
    # of z (z rounding moves the grid by at most s/2)
    assert np.all(err <= np.repeat(s, G, axis=1) * 1.0 + 1e-12)


def _fc_pin_holds(fc, B):
    codes = np.arange(2 ** B)
    for k in range(1, B + 1):
        qh = fc(codes, B, k)
        d = B - k
        if k == B and not np.array_equal(qh, codes.astype(np.float64)):
            return False
        if Fraction(sum(Fraction(float(c)) - Fraction(float(h)) for c, h in zip(codes, qh))) != 0:
            return False
        if np.max(np.abs(codes - qh)) != (2 ** d - 1) / 2:
            return False
        # 2*q_hat = top k bits, then a 0, then (B-k) ones
        twice = (2 * qh).astype(np.int64)
        want = ((codes >> d) << (d + 1)) | ((1 << d) - 1)
        if not np.array_equal(twice, want):
            return False
    return True


@pytest.mark.parametrize("B", [2, 3, 4, 5])
def test_floor_and_compensation_closed_forms(B):
    assert _fc_pin_holds(O.fc_code, B)


def test_planted_floor_without_compensation_fails_the_pin():
    def plain_floor(q, B, k):       # the ablation the MatMoE review reports at 0% accuracy
        d = B - k
        return (np.asarray(q) >> d).astype(np.float64) * 2 ** d
    assert not _fc_pin_holds(plain_floor, 4)
    codes = np.arange(16)
    for k in range(1, 4):
        assert np.mean(codes - plain_floor(codes, 4, k)) == (2 ** (4 - k) - 1) / 2


def test_bitplane_round_trip_and_prefix():
    rng = np.random.default_rng(1)
    q = rng.integers(0, 16, size=(5, 64))
    pl = O.bitplanes(q, 4)
    assert pl.shape == (4, 5, 64)
    assert np.array_equal(pl[0], q >> 3) and np.array_equal(pl[3], q & 1)
    for k in range(1, 5):
        assert np.array_equal(O.codes_from_planes(pl, k, 4), (q >> (4 - k)) << (4 - k))
        # F&C from the prefix alone equals F&C from the full code
        fc_prefix = O.codes_from_planes(pl, k, 4).astype(np.float64) + (2 ** (4 - k) - 1) / 2
        assert np.array_equal(fc_prefix, O.fc_code(q, 4, k))


# ----------------------------------------------------------------- residual table

def test_residual_table_exact_small():
    rng = np.random.default_rng(3)
    H, I, G, B = 16, 8, 8, 4
    g = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
    u = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
    d = (rng.standard_normal((H, I)) * 0.02).astype(np.float32)
    enc = O.encode_expert(g, u, d, 0, B, G)
    for k in range(1, B + 1):
        exact = Fraction(0)
        for m, q, s, z in zip((g, u, d), enc["q"], enc["s"], enc["z"]):
            R, C = m.shape
            for i in range(R):
                for j in range(C):
                    qq = int(q[i, j])
                    dd = B - k
                    qh = Fraction((qq >> dd) << dd) + Fraction(2 ** dd - 1, 2)
                    wh = Fraction(float(s[i, j // G])) * (qh - Fraction(float(z[i, j // G])))
                    diff = Fraction(float(m[i, j])) - wh
                    exact += diff * diff
        assert abs(Fraction(enc["r"][k - 1]) - exact) <= exact * Fraction(1, 10 ** 12), k


def test_residual_table_four_per_plane_uniform():
    rng = np.random.default_rng(5)
    H, I, G, B = 256, 128, 64, 4
    mats = [(rng.standard_normal(sh) * 0.02).astype(np.float32) for sh in ((I, H), (I, H), (H, I))]
    r = O.encode_expert(*mats, 0, B, G)["r"]
    assert np.all(np.diff(r) < 0)
    # dropping one more uniform bit multiplies the mean squared error by ~4 (closed form
    # (4^d/4 - 1/4 + 1/12)/(4^(d-1)/4 - 1/4 + 1/12) -> 4); clamping makes it approximate
    for k in range(1, B):
        assert 3.3 < r[k - 1] / r[k] < 4.7, (k, r)


def test_bcq_closed_forms():
    G = 8
    c = 0.0234375   # exactly representable in fp16
    pattern = np.array([1, -1, -1, 1, 1, 1, -1, 1], dtype=np.float64)
    w = (c * pattern).astype(np.float32)[None, :]
    signs, alpha = O.encode_bcq_matrix(w, 3, G)
    assert alpha[0, 0, 0] == c and alpha[1, 0, 0] == 0.0 and alpha[2, 0, 0] == 0.0
    assert np.array_equal(signs[0, 0], pattern > 0)
    assert np.all(signs[1, 0])        # residual is exactly 0 -> sign(0) = +1
    # random: alpha_0 = fp16(mean |w|) computed exactly; residual non-increasing in k
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((4, 32)) * 0.02).astype(np.float32)
    signs, alpha = O.encode_bcq_matrix(w, 3, 16)
    for r_ in range(4):
        for gi in range(2):
            seg = w[r_, gi * 16:(gi + 1) * 16]
            m = sum(Fraction(abs(float(v))) for v in seg) / 16
            assert Fraction(alpha[0, r_, gi]) == rne_to_format(m, 10, -14)
            # least squares optimum for the chosen signs is the unrounded mean |R|
    prev = np.inf
    for k in range(1, 4):
        e = np.sum((w.astype(np.float64) - O.dequant_bcq(signs, alpha, k, 16)) ** 2)
        assert e <= prev
        prev = e


def _golden_bcq():
    fx = json.load(open(os.path.join(GOLDEN, "bcq_worked_group.json")))
    u = fx["unit"]
    w = np.array(fx["w_units"], dtype=np.float64) * u
    return fx, u, w


def _bcq_pin_holds(encode, dequant):
    """The hand-worked group: exact signs, alphas, w_hat(k) and squared residuals."""
    fx, u, w = _golden_bcq()
    B, G = fx["B"], fx["G"]
    signs, alpha = encode(w.astype(np.float32)[None, :], B, G)
    if not np.array_equal(signs[:, 0, :].astype(int), np.array(fx["signs"])):
        return False
    if [float(a) for a in alpha[:, 0, 0]] != [a * u for a in fx["alpha_units"]]:
        return False
    for k in range(1, B + 1):
        wh = dequant(signs, alpha, k, G)[0]
        if wh.tolist() != [v * u for v in fx["w_hat_units"][str(k)]]:
            return False
        if float(np.sum((w - wh) ** 2)) != fx["r_units2"][str(k)] * u * u:
            return False
    return True


def test_bcq_hand_worked_group_exact():
    assert _bcq_pin_holds(O.encode_bcq_matrix, O.dequant_bcq)


def test_planted_bcq_mistakes_fail_the_pin():
    def sign_swap_after_first(signs, alpha, k, G):      # b = -1 for a set bit on planes >= 1
        B, R, C = signs.shape
        out = np.zeros((R, C))
        for i in range(k):
            b = np.where(signs[i], 1.0, -1.0) * (1.0 if i == 0 else -1.0)
            out = out + np.repeat(alpha[i], G, axis=1) * b
        return out

    def alpha_of_previous_plane(signs, alpha, k, G):    # plane i scaled by alpha_{i-1}
        B, R, C = signs.shape
        out = np.zeros((R, C))
        for i in range(k):
            out = out + np.repeat(alpha[max(i - 1, 0)], G, axis=1) * np.where(signs[i], 1.0, -1.0)
        return out

    def one_plane_short(signs, alpha, k, G):            # dropped last term
        return O.dequant_bcq(signs, alpha, k - 1, G) if k > 1 else np.zeros(signs.shape[1:])

    def refit_sign_of_zero_negative(w, B, G):           # sign(0) = -1 instead of +1
        R, C = w.shape
        res = np.asarray(w, np.float64).reshape(R, C // G, G).copy()
        signs = np.empty((B, R, C // G, G), dtype=bool)
        alpha = np.empty((B, R, C // G))
        for i in range(B):
            pos = res > 0.0
            a = O.fp16_round(np.abs(res).sum(-1) / G)
            res = res - a[..., None] * np.where(pos, 1.0, -1.0)
            signs[i], alpha[i] = pos, a
        return signs.reshape(B, R, C), alpha

    for bad in (sign_swap_after_first, alpha_of_previous_plane, one_plane_short):
        assert not _bcq_pin_holds(O.encode_bcq_matrix, bad), bad.__name__
    # the sign(0) reading shows on a group whose residual reaches exactly 0
    c = 0.0234375
    w = (c * np.array([1, -1, -1, 1, 1, 1, -1, 1], dtype=np.float64)).astype(np.float32)[None, :]
    s_good, _ = O.encode_bcq_matrix(w, 3, 8)
    s_bad, _ = refit_sign_of_zero_negative(w, 3, 8)
    assert np.all(s_good[1]) and not np.array_equal(s_good, s_bad)


def _exact_greedy_bcq(row_group, B):
    """Greedy binary-coded fit of one group in exact rational arithmetic: signs (True = +1),
    alphas (fp16-rounded exact means) and the exact squared residual after each plane."""
    R = [Fraction(float(v)) for v in row_group]
    G = len(R)
    signs, alphas, res2 = [], [], []
    for _ in range(B):
        b = [r >= 0 for r in R]
        a = rne_to_format(sum(abs(r) for r in R) / G, 10, -14)
        R = [r - a if bb else r + a for r, bb in zip(R, b)]
        signs.append(b)
        alphas.append(a)
        res2.append(sum(r * r for r in R))
    return signs, alphas, res2


def test_bcq_fit_and_residual_table_exact_random():
    # values on a 2^-24 grid below 0.1 in magnitude: the exact greedy fit and the oracle's fp64
    # fit take the same steps, and every residual and sum of squares is exact in fp64
    rng = np.random.default_rng(31)
    H, I, G, B = 16, 8, 8, 3
    mats = [np.clip(np.round(rng.standard_normal(sh) * 0.02 * 2.0 ** 24) / 2.0 ** 24, -0.09, 0.09).astype(np.float32)
            for sh in ((I, H), (I, H), (H, I))]
    enc = O.encode_expert(*mats, 1, B, G)
    total = [Fraction(0)] * B
    for m, sg, al in zip(mats, enc["signs"], enc["alpha"]):
        Rr, C = m.shape
        for i in range(Rr):
            for gi in range(C // G):
                signs, alphas, res2 = _exact_greedy_bcq(m[i, gi * G:(gi + 1) * G], B)
                for p in range(B):
                    assert Fraction(float(al[p, i, gi])) == alphas[p]
                    assert sg[p, i, gi * G:(gi + 1) * G].tolist() == signs[p]
                    total[p] += res2[p]
    for k in range(1, B + 1):
        assert Fraction(float(enc["r"][k - 1])) == total[k - 1], k


# ----------------------------------------------------------------- exp

def _cr_exp(x: float) -> float:
    getcontext().prec = 60
    v = Decimal(x).exp()
    return float(Fraction(v))   # float(Fraction) rounds correctly


def test_dexp_within_one_ulp_of_correctly_rounded():
    rng = np.random.default_rng(11)
    xs = list(-rng.random(1500) * 50.0) + list(-rng.random(300) * 700.0) + \
        [0.0, -1e-300, -2.0 ** -60, -0.5 * math.log(2), -math.log(2), -1.0, -707.9, -708.0, -30.0]
    for x in xs:
        got = O.dexp(x)
        want = _cr_exp(x)
        assert abs(got - want) <= f64_ulp(want), (x, got, want)
    assert O.dexp(0.0) == 1.0
    assert O.dexp(-709.0) == 0.0
    s = sorted(xs)
    vals = [O.dexp(x) for x in s]
    assert all(a <= b for a, b in zip(vals, vals[1:]))


def test_exp_constants_from_ln2():
    getcontext().prec = 60
    ln2 = Fraction(Decimal(2).ln())
    assert Fraction(O.LN2_HI) <= ln2 < Fraction(O.LN2_HI) + Fraction(1, 2 ** 42)
    assert (Fraction(O.LN2_HI) * 2 ** 42).denominator == 1
    assert abs(Fraction(O.LN2_HI) + Fraction(O.LN2_LO) - ln2) < Fraction(1, 2 ** 100)
    assert O.INV_LN2 == float(1 / ln2)
    assert all(Fraction(c) == rne_to_format(Fraction(1, math.factorial(i)), 52, -1022)
               for i, c in enumerate(O.EXP_TAYLOR))


# ----------------------------------------------------------------- router

def _bf16_bits(vals):
    from dynamic_any_precision_b200.workloads import f32_to_bf16_bits
    return f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


def test_router_logit_is_exact_dot_rounded_once():
    rng = np.random.default_rng(13)
    T, E, H = 3, 5, 64
    # wide exponent range (incl. values near bf16's subnormal end) so that a naive
    # left-to-right fp64 sum would round differently
    x = rng.standard_normal((T, H)) * np.exp2(rng.integers(-60, 30, size=(T, H)))
    w = rng.standard_normal((E, H)) * np.exp2(rng.integers(-60, 30, size=(E, H)))
    xb, wb = _bf16_bits(x), _bf16_bits(w)
    logits = O.router_logits(xb, wb)
    xf, wf = O.bf16_bits_to_f64(xb), O.bf16_bits_to_f64(wb)
    for t in range(T):
        for e in range(E):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[t], wf[e]))
            assert Fraction(logits[t, e]) == rne_to_format(exact, 52, -1022)


def test_topk_brute_force_ties_and_permutation():
    row = np.array([0.5, 1.0, 1.0, -2.0, 0.75, 1.0])
    assert O.topk_select(row, 3) == [1, 2, 5]
    assert O.topk_select(row, 4) == [1, 2, 5, 4]
    rng = np.random.default_rng(17)
    T, E, H, K = 4, 16, 32, 4
    xb = _bf16_bits(rng.standard_normal((T, H)))
    wb = _bf16_bits(rng.standard_normal((E, H)) * 0.02)
    idx, g, lg = O.route(xb, wb, K, 1)
    for t in range(T):
        brute = sorted(range(E), key=lambda e: -lg[t, e])[:K]
        assert idx[t].tolist() == brute
    perm = rng.permutation(E)
    idx2, g2, _ = O.route(xb, wb[perm], K, 1)
    assert np.array_equal(perm[idx2], idx) and np.array_equal(g2, g)


def test_gate_identities():
    rng = np.random.default_rng(19)
    T, E, H, K = 3, 12, 32, 4
    xb = _bf16_bits(rng.standard_normal((T, H)))
    wb = _bf16_bits(rng.standard_normal((E, H)) * 0.3)
    for norm in (0, 1):
        idx, g, lg = O.route(xb, wb, K, norm)
        for t in range(T):
            sel = idx[t]
            full = np.exp(lg[t] - lg[t].max())
            den = full[sel].sum() if norm else full.sum()
            np.testing.assert_allclose(g[t], full[sel] / den, rtol=1e-13)
            if norm:
                assert abs(g[t].sum() - 1.0) < 1e-15 * K
            assert np.all(np.diff(g[t]) <= 0)


# ----------------------------------------------------------------- allocation

def _tiny_alloc_case(seed, T=4, K=2, E=8, B=4):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    g = rng.dirichlet(np.ones(K), size=T)
    g = -np.sort(-g, axis=1)
    base = rng.random(E) * 10 + 1
    r = np.stack([base * 4.0 ** (B - k) * (1 + 0.3 * rng.random(E)) for k in range(1, B + 1)], axis=1)
    return idx, g, r


@pytest.mark.parametrize("seed,target", [(0, 3.0), (1, 2.5), (2, 2.125), (3, 3.75), (4, 3.0)])
def test_allocation_matches_brute_force_optimum(seed, target):
    kmin, kmax = 2, 4
    idx, g, r = _tiny_alloc_case(seed)
    k, lam = O.allocate(idx, g, r, kmin, kmax, target)
    P = idx.size
    e, gg = idx.reshape(-1), g.reshape(-1)
    n_hi = int(k.sum())
    assert n_hi <= target * P
    def obj(kv):
        return sum(Fraction(float(gg[p])) * Fraction(float(r[e[p], kv[p] - 1])) for p in range(P))
    best, best_set = None, []
    for kv in itertools.product(range(kmin, kmax + 1), repeat=P):
        if sum(kv) > n_hi:
            continue
        o = obj(kv)
        if best is None or o < best:
            best, best_set = o, [kv]
        elif o == best:
            best_set.append(kv)
    assert tuple(k.reshape(-1).tolist()) in best_set
    # generic case: within one plane-step of the budget
    assert n_hi > target * P - 1


def test_allocation_endpoints_and_monotone_trace():
    idx, g, r = _tiny_alloc_case(5, T=6, K=3)
    k, _ = O.allocate(idx, g, r, 2, 4, 2.0)
    assert np.all(k == 2)
    k, _ = O.allocate(idx, g, r, 2, 4, 4.0)
    assert np.all(k == 4)
    trace = []
    O.allocate(idx, g, r, 2, 4, 3.0, trace=trace)
    assert len(trace) == 64
    srt = sorted(trace)
    assert all(a[1] >= b[1] for a, b in zip(srt, srt[1:]))   # N(lambda) non-increasing
    with pytest.raises(ValueError):
        O.allocate(idx, g, r, 2, 4, 4.5)


def test_allocation_prefers_high_gate_pairs():
    # two pairs on the same expert, one with a larger gate: at a budget that allows one
    # extra plane, the larger gate gets it
    idx = np.array([[0, 1], [0, 1]], dtype=np.int32)
    g = np.array([[0.9, 0.1], [0.6, 0.4]])
    r = np.array([[64.0, 16.0, 4.0, 1.0], [64.0, 16.0, 4.0, 1.0]])
    k, lam = O.allocate(idx, g, r, 2, 4, 2.25)
    assert k.tolist() == [[3, 2], [2, 2]]


# ----------------------------------------------------------------- allocation policies

@pytest.mark.parametrize("P,target", [(8, 3.0), (8, 2.5), (7, 2.2), (512, 3.1), (96, 2.0), (1, 3.999)])
def test_uniform_allocation_closed_form(P, target):
    kmin, kmax = 2, 4
    k = O.allocate_uniform(P, kmin, kmax, target)
    total = int(Fraction(target) * P)                      # floor of the exact budget
    assert int(k.sum()) == total and k.max() - k.min() <= 1
    assert np.all((k >= kmin) & (k <= kmax))
    assert np.all(np.diff(k) <= 0)                        # the extra planes go to the first pairs
    if float(target).is_integer():
        assert np.all(k == int(target))


def _brute_force_threshold_count(scores, kmin, kmax, target):
    """Largest high set of the form {s > v} (v = 0 or a score) whose average fits the target."""
    n = len(scores)
    best = 0
    for v in [0.0] + list(scores):
        m = sum(1 for s in scores if s > v)
        if Fraction(kmin * n + (kmax - kmin) * m) <= Fraction(target) * n:
            best = max(best, m)
    return best


@pytest.mark.parametrize("seed,target,kmin,kmax", [(0, 3.0, 2, 4), (1, 2.5, 2, 4), (2, 1.7, 1, 3), (3, 3.9, 2, 4),
                                                   (4, 2.0, 2, 4), (5, 4.0, 2, 4), (6, 2.2, 2, 3)])
def test_threshold_calibration_matches_brute_force(seed, target, kmin, kmax):
    rng = np.random.default_rng(seed)
    scores = rng.dirichlet(np.ones(8), size=6).reshape(-1)       # 48 gate-like scores in (0, 1)
    scores[5] = scores[7]                                        # a tie
    tau = O.calibrate_threshold(scores, kmin, kmax, target)
    k = O.allocate_threshold(scores, tau, kmin, kmax)
    assert Fraction(int(k.sum())) <= Fraction(target) * scores.size
    assert int(np.count_nonzero(k == kmax)) == _brute_force_threshold_count(scores.tolist(), kmin, kmax, target)
    if target == kmin:
        assert np.all(k == kmin)
    if target == kmax:
        assert np.all(k == kmax)
    trace = []
    O.calibrate_threshold(scores, kmin, kmax, target, trace=trace)
    srt = sorted(trace)
    assert len(trace) == 64 and all(a[1] >= b[1] for a, b in zip(srt, srt[1:]))


def test_two_plane_lagrangian_with_equal_residuals_is_a_score_threshold():
    # with two plane counts and the same residuals for every expert, pair p reads kmax exactly
    # when g_p (r(kmin) - r(kmax)) > lambda: a threshold on the gate. The Lagrangian allocation of
    # a batch then equals the threshold policy calibrated on that batch's own gates.
    rng = np.random.default_rng(12)
    T, K, E = 16, 4, 16
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    g = -np.sort(-rng.dirichlet(np.ones(K), size=T), axis=1)
    r = np.tile(np.array([64.0, 16.0, 4.0, 1.0]), (E, 1))
    for target in (2.25, 2.5, 2.8):
        k_lag, _ = O.allocate(idx, g, r, 2, 3, target)
        tau = O.calibrate_threshold(g, 2, 3, target)
        assert np.array_equal(O.allocate_threshold(g, tau, 2, 3), k_lag), target


def test_moe_forward_policies_use_their_plane_counts():
    shape, experts, xb, wb = _mini_layer(25)
    y_u, aux_u = O.moe_forward(xb, wb, experts, shape, 2.5, policy=O.ALLOC_UNIFORM)
    assert aux_u["k"].reshape(-1).tolist() == O.allocate_uniform(6, 2, 4, 2.5).tolist()
    y_t, aux_t = O.moe_forward(xb, wb, experts, shape, 3.0, policy=O.ALLOC_THRESHOLD, threshold=0.5)
    assert np.array_equal(aux_t["k"], np.where(aux_t["gates"] > 0.5, 4, 2))
    assert aux_t["lambda"] == 0.5


# ----------------------------------------------------------------- workload-profiled read rates

def test_distortion_tensor_channels_sum_to_the_gate_up_residual():
    rng = np.random.default_rng(51)
    H, I, G, B = 64, 16, 16, 4
    g = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
    u = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
    d = (rng.standard_normal((H, I)) * 0.02).astype(np.float32)
    for fmt, bb in ((0, B), (1, 3)):
        enc = O.encode_expert(g, u, d, fmt, bb, G)
        T = O.distortion_tensor(enc, fmt, bb, G, g, u)
        for k in range(1, bb + 1):
            wg, wu, _ = O.dequant_expert(enc, fmt, bb, k, G)
            exact = [sum((Fraction(float(gm[i, j])) - Fraction(float(wm[i, j]))) ** 2
                         for gm, wm in ((g, wg), (u, wu)) for i in range(I)) for j in range(H)]
            for j in range(H):
                assert abs(Fraction(T[k - 1, j]) - exact[j]) <= exact[j] * Fraction(1, 10 ** 12)
        # monotone in k for uniform codes (each extra plane halves the step)
        if fmt == 0:
            assert np.all(T[:-1].sum(axis=1) > T[1:].sum(axis=1))


def test_prefill_profile_exact_and_counts():
    rng = np.random.default_rng(52)
    x = _bf16_bits(rng.standard_normal((5, 32)))
    idx = np.array([[0, 3], [3, 1], [0, 3], [2, 0], [3, 1]])
    m, c = O.prefill_profile(x, idx, 6)
    xf = O.bf16_bits_to_f64(x)
    for j in range(32):
        exact = sum(Fraction(float(xf[t, j])) ** 2 for t in range(5)) / 5
        assert abs(Fraction(m[j]) - exact) <= exact * Fraction(1, 10 ** 14)
    assert c.tolist() == [3, 2, 1, 4, 0, 0]


def test_tree_dot_order_and_accuracy():
    rng = np.random.default_rng(53)
    m = rng.random(64) * 3
    t = rng.random(64) * 1e-3
    v = O.tree_dot(m, t)
    exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(m, t))
    assert abs(Fraction(v) - exact) <= abs(exact) * Fraction(8, 2 ** 53)
    # the chunk/tree order: a value in chunk 0 and its negative in chunk 16 cancel at the first
    # tree level, so a 1 in chunk 1 survives (a left-to-right sum would lose it)
    m2 = np.ones(64)
    t2 = np.zeros(64)
    t2[0], t2[32], t2[2] = 1e17, -1e17, 1.0
    assert O.tree_dot(m2, t2) == 1.0
    seq = 0.0
    for v in t2:
        seq = seq + v
    assert seq == 0.0


def _rates_case(seed, E=5, B=4, H=32):
    rng = np.random.default_rng(seed)
    base = rng.random((E, 1)) * 5 + 0.5
    T = np.stack([base * 4.0 ** (B - k) * (1 + 0.2 * rng.random((E, H))) for k in range(1, B + 1)], axis=1)
    m = rng.random(H) + 0.1
    counts = rng.integers(0, 6, size=E)
    counts[0] = max(counts[0], 1)
    return T, m, counts


@pytest.mark.parametrize("seed,target", [(0, 3.0), (1, 2.5), (2, 3.6), (3, 2.2), (4, 4.0), (5, 2.0)])
def test_expert_rates_match_brute_force_and_frequency_cancels(seed, target):
    kmin, kmax = 2, 4
    T, m, counts = _rates_case(seed)
    k, lam, D = O.solve_expert_rates(T, m, counts, kmin, kmax, target)
    n_hi = int(np.sum(counts * k))
    assert n_hi <= target * counts.sum()
    if target in (kmin, kmax):
        assert np.all(k[counts > 0] == target)
    # the count-weighted objective is minimal among all tables that read at most as many planes
    best, best_set = None, []
    for kv in itertools.product(range(kmin, kmax + 1), repeat=len(k)):
        if sum(c * kk for c, kk in zip(counts, kv)) > n_hi:
            continue
        o = sum(Fraction(int(c)) * Fraction(float(D[e, kk - kmin])) for e, (c, kk) in enumerate(zip(counts, kv)))
        if best is None or o < best:
            best, best_set = o, [kv]
        elif o == best:
            best_set.append(kv)
    used = counts > 0
    assert any(all(a == b for a, b, u in zip(k.tolist(), bs, used) if u) for bs in best_set)
    # frequency cancels: scaling every count by 3 leaves the solution unchanged
    k3, lam3, _ = O.solve_expert_rates(T, m, counts * 3, kmin, kmax, target)
    assert np.array_equal(k3, k) and lam3 == lam


def test_expert_rate_table_allocation():
    idx = np.array([[0, 2], [1, 2]])
    assert O.allocate_expert_table(idx, np.array([4, 2, 3])).tolist() == [[4, 3], [2, 3]]


# ----------------------------------------------------------------- FFN and combine

def test_expert_ffn_hand_worked():
    x = np.array([1.0, 2.0])
    wg = np.array([[0.5, 0.25]])
    wu = np.array([[1.0, -1.0]])
    wd = np.array([[2.0], [-4.0]])
    o = O.expert_ffn(x, wg, wu, wd)
    s1 = 1.0 / (1.0 + math.exp(-1.0))          # silu(1) = 1 * sigmoid(1); a = 1, u = -1
    np.testing.assert_allclose(o, [-2.0 * s1, 4.0 * s1], rtol=1e-15)
    # swapping gate and up gives a = -1, u = 1 -> a different value (catches a swap)
    o2 = O.expert_ffn(x, wu, wg, wd)
    assert not np.allclose(o, o2)


def _mini_layer(seed, fmt=0, K=2, norm=1, B=4, kmin=2, kmax=4):
    from dynamic_any_precision_b200.workloads import LayerShape
    shape = LayerShape("mini", 32, 16, 4, K, 0, fmt, B, kmin, kmax, 16, norm, 3, (3.0,), seed)
    rng = np.random.default_rng(seed)
    experts = {}
    for e in range(4):
        mats = [(rng.standard_normal(sh) * 0.2).astype(np.float32) for sh in ((16, 32), (16, 32), (32, 16))]
        experts[e] = O.encode_expert(*mats, fmt, B, 16)
    xb = _bf16_bits(rng.standard_normal((3, 32)))
    wb = _bf16_bits(rng.standard_normal((4, 32)))
    return shape, experts, xb, wb


def test_moe_combine_is_gate_weighted_sum_and_top1_identity():
    shape, experts, xb, wb = _mini_layer(21)
    y, aux = O.moe_forward(xb, wb, experts, shape, 3.0)
    x = O.bf16_bits_to_f64(xb)
    for t in range(3):
        acc = np.zeros(32)
        for j in range(2):
            e, k = int(aux["idx"][t, j]), int(aux["k"][t, j])
            wg, wu, wd = O.dequant_expert(experts[e], 0, 4, k, 16)
            acc += aux["gates"][t, j] * O.expert_ffn(x[t], wg, wu, wd)
        np.testing.assert_allclose(y[t], acc, rtol=1e-14, atol=1e-15)
    shape1, experts1, xb1, wb1 = _mini_layer(22, K=1)
    y1, aux1 = O.moe_forward(xb1, wb1, experts1, shape1, 3.0)
    assert np.all(aux1["gates"] == 1.0)
    for t in range(3):
        e, k = int(aux1["idx"][t, 0]), int(aux1["k"][t, 0])
        wg, wu, wd = O.dequant_expert(experts1[e], 0, 4, k, 16)
        np.testing.assert_array_equal(y1[t], O.expert_ffn(O.bf16_bits_to_f64(xb1)[t], wg, wu, wd))


def test_prefix_property_low_bits_ignored():
    shape, experts, xb, wb = _mini_layer(23)
    y, aux = O.moe_forward(xb, wb, experts, shape, 2.0)     # every pair reads k = 2 planes
    assert np.all(aux["k"] == 2)
    rng = np.random.default_rng(0)
    poisoned = {}
    for e, enc in experts.items():
        enc2 = dict(enc)
        enc2["q"] = [((q >> 2) << 2) | rng.integers(0, 4, size=q.shape).astype(np.uint8) for q in enc["q"]]
        poisoned[e] = enc2
    y2, _ = O.moe_forward(xb, wb, poisoned, shape, 2.0, r_table=np.stack([experts[e]["r"] for e in range(4)]))
    np.testing.assert_array_equal(y, y2)


def test_bcq_moe_runs_and_shared_expert_adds():
    shape, experts, xb, wb = _mini_layer(24, fmt=1, B=3, kmin=1, kmax=3, norm=0)
    y, aux = O.moe_forward(xb, wb, experts, shape, 2.0)
    assert np.all(np.isfinite(y))
    rng = np.random.default_rng(1)
    sh = (_bf16_bits(rng.standard_normal((1, 16, 32)) * 0.1), _bf16_bits(rng.standard_normal((1, 16, 32)) * 0.1),
          _bf16_bits(rng.standard_normal((1, 32, 16)) * 0.1))
    y2, _ = O.moe_forward(xb, wb, experts, shape, 2.0, shared=sh)
    x = O.bf16_bits_to_f64(xb)
    for t in range(3):
        extra = O.expert_ffn(x[t], O.bf16_bits_to_f64(sh[0][0]), O.bf16_bits_to_f64(sh[1][0]),
                             O.bf16_bits_to_f64(sh[2][0]))
        np.testing.assert_allclose(y2[t] - y[t], extra, rtol=1e-12, atol=1e-14)


def _torch_layer_at_full_rate(shape, experts, xb, wb):
    """The layer at k = B with library routines only (torch, CPU): fp64 logits, torch.topk,
    torch.softmax, the textbook dequantisation s*(q - z) or sum_i alpha_i*b_i of the stored
    codes, and fp32 matmuls with torch's silu."""
    import torch
    x64 = torch.from_numpy(O.bf16_bits_to_f64(xb))
    w64 = torch.from_numpy(O.bf16_bits_to_f64(wb))
    logits = x64 @ w64.T
    top, idx = torch.topk(logits, shape.top_k, dim=1)
    if shape.norm_topk:
        gates = torch.softmax(top, dim=1)
    else:
        gates = torch.gather(torch.softmax(logits, dim=1), 1, idx)
    G = shape.group

    def dense(enc, m):
        if shape.fmt == 0:
            q = torch.from_numpy(enc["q"][m].astype(np.float32))
            s = torch.from_numpy(enc["s"][m].astype(np.float32)).repeat_interleave(G, dim=1)
            z = torch.from_numpy(enc["z"][m].astype(np.float32)).repeat_interleave(G, dim=1)
            return s * (q - z)
        sg = torch.from_numpy(enc["signs"][m])
        al = torch.from_numpy(enc["alpha"][m].astype(np.float32)).repeat_interleave(G, dim=2)
        return (al * (sg.float() * 2.0 - 1.0)).sum(dim=0)

    x32 = x64.float()
    y = torch.zeros((xb.shape[0], shape.hidden), dtype=torch.float32)
    for t in range(xb.shape[0]):
        for j in range(shape.top_k):
            enc = experts[int(idx[t, j])]
            wg, wu, wd = dense(enc, 0), dense(enc, 1), dense(enc, 2)
            h = torch.nn.functional.silu(wg @ x32[t]) * (wu @ x32[t])
            y[t] += float(gates[t, j]) * (wd @ h)
    return y.numpy().astype(np.float64), idx.numpy(), gates.numpy()


@pytest.mark.parametrize("fmt", [0, 1])
def test_layer_at_full_rate_matches_torch_library_routines(fmt):
    from dynamic_any_precision_b200.workloads import LayerShape
    B, kmin = (4, 2) if fmt == 0 else (3, 1)
    shape = LayerShape("lib_check", 64, 32, 6, 2, 0, fmt, B, kmin, B, 16, 1 - fmt, 5, (float(B),), 41)
    rng = np.random.default_rng(41 + fmt)
    experts = {}
    for e in range(shape.n_experts):
        mats = [(rng.standard_normal(sh) * 0.1).astype(np.float32) for sh in ((32, 64), (32, 64), (64, 32))]
        experts[e] = O.encode_expert(*mats, fmt, B, 16)
    xb = _bf16_bits(rng.standard_normal((5, 64)))
    wb = _bf16_bits(rng.standard_normal((6, 64)) * 0.3)
    y, aux = O.moe_forward(xb, wb, experts, shape, float(B))
    assert np.all(aux["k"] == B)
    y_t, idx_t, g_t = _torch_layer_at_full_rate(shape, experts, xb, wb)
    assert np.array_equal(aux["idx"], idx_t)
    np.testing.assert_allclose(aux["gates"], g_t, rtol=1e-12, atol=0)
    np.testing.assert_allclose(y, y_t, rtol=2e-5, atol=2e-6)


# ----------------------------------------------------------------- stack glue

def test_rmsnorm_closed_form_and_bf16_rounding():
    v = np.full((2, 8), 3.0)
    np.testing.assert_allclose(O.rmsnorm(v), 3.0 / math.sqrt(9.0 + 1e-6), rtol=1e-15)
    assert np.all(O.rmsnorm(np.zeros((1, 4))) == 0.0)
    vals = [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -30, -2.5, 1e-3, 123.456]
    bits = O.f64_to_bf16_bits(np.array(vals))
    for v_, b in zip(vals, bits):
        got = Fraction(float(np.array([int(b) << 16], dtype=np.uint32).view(np.float32)[0]))
        assert got == rne_to_format(Fraction(v_), 7, -126), v_


# ---- per-expert stored widths (MatMoE, "Core Contribution": offline ILP over 2/3/4-bit
# maximum widths under a memory budget) ----

def _brute_widths(imp, r, kmin, kmax, budget):
    """Lexicographically smallest optimal widths by enumeration (exact: integer data)."""
    import itertools
    best, arg = None, None
    for ws in itertools.product(range(kmin, kmax + 1), repeat=len(imp)):
        if sum(ws) > budget:
            continue
        cost = sum(int(imp[e]) * int(r[e][b - 1]) for e, b in enumerate(ws))
        if best is None or cost < best:
            best, arg = cost, ws
    return np.array(arg, dtype=np.int64)


def test_stored_widths_dp_matches_brute_force():
    rng = np.random.default_rng(11)
    for trial in range(60):
        E = int(rng.integers(1, 5))
        kmin, kmax = (2, 4) if trial % 2 else (1, 3)
        imp = rng.integers(1, 10, size=E).astype(np.float64)
        # residuals: integers, non-increasing in the width but not convex (plane steps of uneven
        # worth), so that a greedy per-step upgrade would not be optimal
        steps = rng.integers(0, 50, size=(E, 4))
        r = np.cumsum(steps[:, ::-1], axis=1)[:, ::-1].astype(np.float64)
        for budget in range(E * kmin, E * kmax + 2):
            got = O.solve_stored_widths(imp, r, kmin, kmax, budget)
            want = _brute_widths(imp, r, kmin, kmax, budget)
            assert np.array_equal(got, want), (trial, budget, got, want)


def test_stored_widths_endpoints_and_budget():
    rng = np.random.default_rng(12)
    imp = rng.random(16) + 0.1
    r = np.sort(rng.random((16, 4)) * 100, axis=1)[:, ::-1].copy()
    assert np.all(O.solve_stored_widths(imp, r, 2, 4, 32) == 2)          # budget = E * kmin
    assert np.all(O.solve_stored_widths(imp, r, 2, 4, 64) == 4)          # budget = E * kmax
    assert np.all(O.solve_stored_widths(imp, r, 2, 4, 1000) == 4)        # more than enough
    prev = None
    for budget in range(32, 65):
        w = O.solve_stored_widths(imp, r, 2, 4, budget)
        assert w.sum() <= budget and np.all((w >= 2) & (w <= 4))
        cost = float(np.sum(imp * r[np.arange(16), w - 1]))
        assert prev is None or cost <= prev + 1e-12                       # more memory never hurts
        prev = cost
    with pytest.raises(ValueError):
        O.solve_stored_widths(imp, r, 2, 4, 31)


def test_routing_mass_is_the_gate_sum_per_expert():
    rng = np.random.default_rng(13)
    idx = np.stack([rng.choice(8, 3, replace=False) for _ in range(20)])
    g = rng.random((20, 3))
    want = np.zeros(8)
    np.add.at(want, idx.reshape(-1), g.reshape(-1))
    assert np.allclose(O.routing_mass(idx, g, 8), want, rtol=0, atol=1e-12)


def test_allocation_respects_stored_widths():
    rng = np.random.default_rng(14)
    E, T, K = 12, 40, 3
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)])
    g = -np.sort(-rng.dirichlet(np.ones(K), size=T), axis=1)
    r = np.sort(rng.random((E, 4)) * 10, axis=1)[:, ::-1].copy()
    cap = rng.integers(2, 5, size=E)
    for target in (2.0, 2.7, 3.4, 4.0):
        k, _ = O.allocate(idx, g, r, 2, 4, target, cap=cap)
        assert np.all(k <= cap[idx]) and np.all(k >= 2)
        assert k.sum() <= target * k.size
        k_full, _ = O.allocate(idx, g, r, 2, 4, target, cap=np.full(E, 4))
        assert np.array_equal(k_full, O.allocate(idx, g, r, 2, 4, target)[0])   # width kmax: no cap
    k_min, _ = O.allocate(idx, g, r, 2, 4, 4.0, cap=np.full(E, 2))
    assert np.all(k_min == 2)
    for pol in (O.ALLOC_UNIFORM, O.ALLOC_THRESHOLD):
        k, _ = O.allocate_policy(pol, idx, g, r, 2, 4, 3.0, threshold=0.3, cap=cap)
        assert np.all(k <= cap[idx])
