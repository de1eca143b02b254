"""CPU models of two decision-path schedules the CUDA kernels use, checked against the oracle's
plain definitions. They test the arguments the kernels rest on, not the kernels (the GPU parity
tests do that):

- the allocation's cluster bisection evaluates a round's tree of midpoints over a pruned list of
  pairs: a pair whose choice is provably the same over the whole current interval adds a fixed
  count. The argument: fl(c_k + fl(lam k)) never decreases as lam grows, so if the choice a at
  hi satisfies fl(c_a + fl(hi a)) < fl(c_b + fl(lo b)) for counts b below a (<= for counts
  above a), the pair chooses a everywhere in [lo, hi]. The model takes the kernel's round
  depths (6, 6, then 8) and prunes once, at the third round; lambda and every count must equal
  the 64-step bisection of the DuoRate page's Lagrangian (Abstract) as the oracle runs it.
- the router's top-k by repeated extraction of the largest order-preserving 64-bit key (-0 as
  +0, NaN lowest), per group of 32 experts and then over the groups' candidates laid out group
  by group, must give the oracle's order: descending logit, ties to the lower expert id.
"""
import math

import numpy as np
import pytest

from oracle import dpa_oracle as O


# ----------------------------------------------------------------------------- allocation

def _midpoint(lo, hi):
    return 0.5 * (lo + hi)


def _choose(c, lam, kmin):
    """Per-pair choice at lam: first minimum of fl(c_k + fl(lam k)) (numpy rounds each op)."""
    ks = np.arange(kmin, kmin + c.shape[1], dtype=np.float64)
    return np.argmin(c + lam * ks[None, :], axis=1) + kmin


def pruned_tree_bisection(c, kmin, target, early=6, late=8, prune_round=2):
    P, nk = c.shape
    ks = np.arange(kmin, kmin + nk, dtype=np.float64)
    nb = math.floor(target * P)
    lo, hi = 0.0, 2.0 * float(np.max(c[:, 0])) + 1.0
    listed = np.arange(P)
    fixed_k = np.zeros(P, dtype=np.int64)
    fixed_sum = 0
    it, rnd = 0, 0
    while it < 64:
        D = min(early if rnd < prune_round else late, 64 - it)
        if rnd == prune_round:
            cl = c[listed]
            vlo = cl + lo * ks[None, :]
            vhi = cl + hi * ks[None, :]
            a = np.argmin(vhi, axis=1)
            va = vhi[np.arange(len(listed)), a]
            same = np.ones(len(listed), dtype=bool)
            for i in range(nk):
                cond = np.where(i < a, va < vlo[:, i], va <= vlo[:, i])
                same &= np.where(i == a, True, cond)
            fixed_k[listed[same]] = a[same] + kmin
            fixed_sum += int((a[same] + kmin).sum())
            listed = listed[~same]
        # every node's midpoint, evaluated over the listed pairs
        nn = (1 << D) - 1
        pred = np.zeros(nn + 1, dtype=np.int64)
        for node in range(1, nn + 1):
            l, h = lo, hi
            for lev in range(node.bit_length() - 2, -1, -1):
                m = _midpoint(l, h)
                if (node >> lev) & 1:
                    l = m
                else:
                    h = m
            n = fixed_sum + int(_choose(c[listed], _midpoint(l, h), kmin).sum())
            pred[node] = 1 if n > nb else 0
        nd = 1
        for _ in range(D):   # the walk on the predicates
            m = _midpoint(lo, hi)
            if pred[nd]:
                lo = m
            else:
                hi = m
            nd = 2 * nd + int(pred[nd])
        it += D
        rnd += 1
    k = fixed_k.copy()
    k[listed] = _choose(c[listed], hi, kmin)
    return k, hi, len(listed)


def _inputs(seed, P, E, B, ties=False):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, E, size=P).astype(np.int32)
    g = rng.random(P)
    if ties:
        g[: P // 2] = g[0]
        idx[: P // 2] = idx[0]
    base = rng.random(E) * 10 + 1
    r = np.stack([base * 4.0 ** (B - k) * (1 + 0.3 * rng.random(E)) for k in range(1, B + 1)], axis=1)
    return idx, g, r


@pytest.mark.parametrize("P,E,kmin,kmax,target,ties,capped", [
    (512, 128, 2, 4, 3.0, False, False), (512, 128, 2, 4, 2.5, False, False), (512, 128, 2, 4, 3.5, True, False),
    (96, 64, 1, 3, 2.0, False, False), (800, 128, 1, 4, 1.7, False, False), (72, 128, 2, 4, 2.2, False, False),
    (512, 128, 2, 4, 4.0, False, False), (512, 128, 2, 4, 2.0, False, False), (256, 128, 2, 4, 2.6, False, True)])
def test_pruned_tree_bisection_matches_the_oracle(P, E, kmin, kmax, target, ties, capped):
    idx, g, r = _inputs(P * 7 + E, P, E, kmax, ties)
    cap = np.random.default_rng(P).integers(kmin, kmax + 1, size=E) if capped else None
    rk, rlam = O.allocate(idx, g, r, kmin, kmax, target, cap=cap)
    c = O.pair_costs(idx, g, r, kmin, kmax, cap)
    k, lam, n_listed = pruned_tree_bisection(c, kmin, target)
    assert lam == rlam
    assert np.array_equal(k, rk.reshape(-1))
    if not ties:
        assert n_listed < P // 4   # the pruning leaves few pairs to evaluate


def test_pruning_rule_is_sound_pair_by_pair():
    # Exhaustive check of the sufficient condition on small random intervals: whenever it
    # declares a pair's choice constant over [lo, hi], the choice at many points inside agrees.
    rng = np.random.default_rng(11)
    ks = np.arange(2, 5, dtype=np.float64)
    for _ in range(300):
        c = np.sort(rng.random(3) * rng.choice([1e-3, 1.0, 1e3]))[::-1].copy()
        lo = rng.random() * 2.0
        hi = lo + rng.choice([1e-12, 1e-6, 1e-2, 1.0]) * rng.random()
        vlo, vhi = c + lo * ks, c + hi * ks
        a = int(np.argmin(vhi))
        same = all((vhi[a] < vlo[i]) if i < a else (vhi[a] <= vlo[i]) for i in range(3) if i != a)
        if same:
            for lam in np.linspace(lo, hi, 33):
                assert int(np.argmin(c + lam * ks)) == a


# ----------------------------------------------------------------------------- top-k

def _key(v):
    if v != v:
        return 0
    b = np.array([0.0 if v == 0.0 else v], dtype=np.float64).view(np.uint64)[0]
    b = int(b)
    return (~b) & 0xFFFFFFFFFFFFFFFF if b >> 63 else b | 0x8000000000000000


def _extract(keys, avail, K):
    """K largest keys among the available slots, equal keys to the lowest slot."""
    out = []
    avail = list(avail)
    for _ in range(K):
        best = -1
        for i, (k, ok) in enumerate(zip(keys, avail)):
            if ok and (best < 0 or k > keys[best]):
                best = i
        if best < 0:
            break
        out.append(best)
        avail[best] = False
    return out


def warp_topk(logits, K):
    E = len(logits)
    keys = [_key(float(v)) for v in logits]
    cand = []
    for w in range((E + 31) // 32):
        ids = list(range(32 * w, min(E, 32 * w + 32)))
        for j in _extract([keys[e] for e in ids], [True] * len(ids), K):
            cand.append(ids[j])
    return [cand[j] for j in _extract([keys[e] for e in cand], [True] * len(cand), K)]


@pytest.mark.parametrize("E,K,seed", [(128, 8, 0), (64, 6, 1), (8, 2, 2), (100, 3, 3)])
def test_warp_extraction_topk_matches_the_oracle_order(E, K, seed):
    rng = np.random.default_rng(seed)
    for trial in range(40):
        v = rng.standard_normal(E) * rng.choice([1e-3, 1.0, 1e6])
        # ties, signed zeros, infinities and NaN
        v[rng.integers(0, E, size=E // 4)] = v[rng.integers(0, E)]
        if trial % 5 == 0:
            v[rng.integers(0, E)] = -0.0
            v[rng.integers(0, E)] = 0.0
        if trial % 7 == 0:
            v[rng.integers(0, E)] = np.inf
            v[rng.integers(0, E)] = -np.inf
        if trial % 9 == 0:
            v[rng.integers(0, E, size=3)] = np.nan
        want = O.topk_select(v, K) if not np.isnan(v).any() else sorted(
            range(E), key=lambda e: (1, e) if np.isnan(v[e]) else (0, -float(v[e]), e))[:K]
        assert warp_topk(v, K) == want, (trial, v)
