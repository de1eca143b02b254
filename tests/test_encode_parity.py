"""Host encoder (C++, product) against the fp64 oracle: codes, scales/zeros or BCQ alphas, and
the residual table must be bit-identical. CPU only."""
import numpy as np
import pytest

from dynamic_any_precision_b200 import dpa, workloads as W
from oracle import dpa_oracle as O


def _check(shape, experts):
    d = dpa.make_desc(shape)
    ws = [W.expert_weights(shape, e) for e in experts]
    g = np.stack([w[0] for w in ws])
    u = np.stack([w[1] for w in ws])
    dn = np.stack([w[2] for w in ws])
    planes, meta, r = None, None, None
    # encode each expert at its own index to exercise e_begin
    out = None
    for i, e in enumerate(experts):
        out = dpa.encode(d, g[i:i + 1], u[i:i + 1], dn[i:i + 1], e_begin=e, out=out)
    planes, meta, r = out
    for i, e in enumerate(experts):
        enc = O.encode_expert(g[i], u[i], dn[i], shape.fmt, shape.bits, shape.group)
        assert np.array_equal(enc["r"], r[e]), (e, enc["r"], r[e])
        for m in range(3):
            codes = dpa.export_codes(d, planes, e, m)
            if shape.fmt == W.FMT_UNIFORM:
                assert np.array_equal(codes, enc["q"][m])
                s, z = dpa.export_meta(d, meta, e, m)
                assert np.array_equal(s.astype(np.float64), enc["s"][m])
                assert np.array_equal(z.astype(np.float64), enc["z"][m])
            else:
                sg = enc["signs"][m]
                want = sum(sg[i_].astype(np.int64) << (shape.bits - 1 - i_) for i_ in range(shape.bits))
                assert np.array_equal(codes, want)
                al, _ = dpa.export_meta(d, meta, e, m)
                assert np.array_equal(al.astype(np.float64), enc["alpha"][m])


def test_tiny_all_experts():
    _check(W.TINY, range(W.TINY.n_experts))


def test_qwen3_shape_two_experts():
    _check(W.QWEN3_B1, [0, 77])


def test_deepseek_bcq_one_expert():
    _check(W.DEEPSEEK_B16, [5])


def test_bcq_small_group64_and_prefix_layout():
    sh = W.with_sizes(W.TINY, fmt=W.FMT_BCQ, bits=3, kmin=1, kmax=3, name="tiny_bcq")
    _check(sh, range(3))


def test_plane_prefix_is_contiguous():
    # the first k planes of a matrix are one contiguous prefix of its bytes: zeroing every
    # byte after that prefix must not change the codes' top k bits
    sh = W.TINY
    d = dpa.make_desc(sh)
    g, u, dn = W.expert_weights(sh, 0)
    planes, meta, r = dpa.encode(d, g[None], u[None], dn[None])
    s = dpa.encoded_sizes(d)
    plane_bytes = sh.inter * sh.hidden // 8
    for k in range(1, sh.bits + 1):
        cut = planes.copy()
        start = s.planes_matrix_offset[0] + k * plane_bytes
        cut[start:s.planes_matrix_offset[1]] = 0xFF if k % 2 else 0x00
        full = dpa.export_codes(d, planes, 0, 0)
        trunc = dpa.export_codes(d, cut, 0, 0)
        sh_ = sh.bits - k
        assert np.array_equal(full >> sh_, trunc >> sh_)


@pytest.mark.parametrize("shape,experts", [(W.TINY, [0, 5]),
                                           (W.with_sizes(W.DEEPSEEK_B16, hidden=256, inter=128, name="bcq_small"), [3])])
def test_distortion_tensor_bit_identical(shape, experts):
    # the baked distortion tensor of the workload-profiled read rates (host C++) against the oracle
    d = dpa.make_desc(shape)
    out = None
    T = None
    for e in experts:
        g, u, dn = W.expert_weights(shape, e)
        out = dpa.encode(d, g[None], u[None], dn[None], e_begin=e, out=out)
    planes, meta, _ = out
    for e in experts:
        g, u, dn = W.expert_weights(shape, e)
        T = dpa.distortion_tensor(d, g[None], u[None], planes, meta, e_begin=e, out=T)
        enc = O.encode_expert(g, u, dn, shape.fmt, shape.bits, shape.group)
        want = O.distortion_tensor(enc, shape.fmt, shape.bits, shape.group, g, u)
        assert np.array_equal(T[e], want), e
