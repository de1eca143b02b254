"""Per-expert stored widths on the host (MatMoE, review "Core Contribution": an offline ILP over
each expert's maximum bit-width under a memory budget): the library's solver is bit-identical to
the oracle's dynamic programme, and the compact layer holds exactly each expert's plane prefix."""
import ctypes

import numpy as np
import pytest

from dynamic_any_precision_b200 import dpa, workloads as W
from oracle import dpa_oracle as O


@pytest.mark.parametrize("E,kmin,kmax,seed", [(8, 2, 4, 0), (128, 2, 4, 1), (64, 1, 3, 2), (16, 1, 4, 3)])
def test_solver_bit_identical_to_oracle(E, kmin, kmax, seed):
    shape = W.with_sizes(W.QWEN3_B1, n_experts=E, kmin=kmin, kmax=kmax, name="w")
    d = dpa.make_desc(shape)
    rng = np.random.default_rng(seed)
    imp = rng.random(E) * rng.integers(1, 4, size=E)
    r = np.sort(rng.random((E, shape.bits)) * 50, axis=1)[:, ::-1].copy()
    imp[rng.integers(0, E)] = 0.0                      # an expert never routed to
    for budget in sorted({E * kmin, E * kmin + 1, (E * (kmin + kmax)) // 2, E * kmax - 1, E * kmax, E * kmax + 7}):
        got = dpa.solve_stored_widths(d, imp, r, budget).astype(np.int64)
        want = O.solve_stored_widths(imp, r, kmin, kmax, budget)
        assert np.array_equal(got, want), budget
        assert got.sum() <= budget


def test_solver_rejects_bad_inputs():
    d = dpa.make_desc(W.TINY)
    imp, r = np.ones(8), np.ones((8, 4))
    with pytest.raises(dpa.DpaError, match="INVALID_ARG"):
        dpa.solve_stored_widths(d, imp, r, 8 * 2 - 1)      # below every expert at kmin
    bad = imp.copy()
    bad[3] = np.nan
    with pytest.raises(dpa.DpaError, match="INVALID_ARG"):
        dpa.solve_stored_widths(d, bad, r, 20)
    bad[3] = -1.0
    with pytest.raises(dpa.DpaError, match="INVALID_ARG"):
        dpa.solve_stored_widths(d, bad, r, 20)


@pytest.mark.parametrize("shape", [W.TINY, W.with_sizes(W.DEEPSEEK_B16, n_experts=6, n_shared=0, name="bcq6")])
def test_compact_layer_holds_each_expert_prefix(shape):
    d = dpa.make_desc(shape)
    g, u, dn = W.all_expert_weights(shape)
    planes, meta, _ = dpa.encode(d, g, u, dn)
    rng = np.random.default_rng(5)
    widths = rng.integers(shape.kmin, shape.kmax + 1, size=shape.n_experts).astype(np.uint8)
    cp, cm, off = dpa.compact_layer(d, planes, meta, widths)
    s = dpa.encoded_sizes(d)
    pb = shape.hidden * shape.inter // 8
    ng_rows = shape.inter * (shape.hidden // shape.group)
    for e in range(shape.n_experts):
        w = int(widths[e])
        p0, m0 = int(off[e][0]), int(off[e][1])
        for m in range(3):
            full = planes[e * s.planes_per_expert + s.planes_matrix_offset[m]:][:w * pb]
            assert np.array_equal(cp[p0 + m * w * pb:][:w * pb], full)
            if shape.fmt == W.FMT_UNIFORM:
                n = ng_rows * 4
                mm = cm[m0 + m * n:][:n]
            else:
                n = w * ng_rows * 2
                mm = cm[m0 + m * n:][:n]
            assert np.array_equal(mm, meta[e * s.meta_per_expert + s.meta_matrix_offset[m]:][:n])
    # fewer bytes than the full layer unless every expert keeps every plane
    assert cp.size == 3 * pb * int(widths.astype(np.int64).sum())
    assert cp.size < planes.size


def test_compact_layer_rejects_bad_widths():
    d = dpa.make_desc(W.TINY)
    w = np.full(8, 3, np.uint8)
    w[2] = 5
    pb, mb = ctypes.c_uint64(0), ctypes.c_uint64(0)
    assert dpa.lib().dpa_compact_sizes(ctypes.byref(d), w.ctypes.data, ctypes.byref(pb), ctypes.byref(mb)) == 1
    w[2] = 1                                           # below kmin = 2
    assert dpa.lib().dpa_compact_sizes(ctypes.byref(d), w.ctypes.data, ctypes.byref(pb), ctypes.byref(mb)) == 1
