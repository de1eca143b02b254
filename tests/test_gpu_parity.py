"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.
Routing indices, gates, plane counts and lambda must be bit-identical; outputs within
|y - y_ref| <= 2e-3 * (1 + |y_ref|)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from dynamic_any_precision_b200 import dpa, workloads as W  # noqa: E402
from oracle import dpa_oracle as O  # noqa: E402
from oracle_jobs import pair_outputs, reference_layer, reference_layer_parallel  # noqa: E402

pytestmark = pytest.mark.gpu
TOL = 2e-3


def half_ulp_bf16(v):
    """Half the spacing of bf16 values at |v| (8 significant bits): the most that rounding an
    exact result to the bf16 output format can move it."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.where(a > 0, np.ldexp(1.0, (e - 8).astype(int)), 0.0)


def within_tol(got, ref, tol=TOL, bf16_out=False):
    """|got - ref| <= tol * (1 + |ref|); for bf16 layer outputs the format's own rounding (half a
    bf16 ulp of ref) comes on top: the fp32 result meets the tolerance, then it is rounded."""
    err = np.abs(got - ref)
    bound = tol * (1.0 + np.abs(ref))
    if bf16_out:
        bound = bound + half_ulp_bf16(ref)
    return bool(np.all(err <= bound)), float(np.max(err / bound))


def bits_to_f64(y_t):
    return O.bf16_bits_to_f64(y_t.cpu().numpy().view(np.uint16))


class GpuLayer:
    """A layer encoded by the product encoder and resident on the GPU."""
    _cache = {}

    @classmethod
    def get(cls, shape):
        if shape.name not in cls._cache:
            cls._cache[shape.name] = cls(shape)
        return cls._cache[shape.name]

    def __init__(self, shape):
        self.shape = shape
        self.desc = dpa.make_desc(shape)
        g, u, d = W.all_expert_weights(shape)
        planes, meta, r = dpa.encode(self.desc, g, u, d)
        del g, u, d
        self.wr = W.router_weights(shape)
        sh = W.shared_weights_bf16(shape) if shape.n_shared else None
        self.layer = dpa.DeviceLayer.from_host(self.desc, planes, meta, r, self.wr, sh)
        self.planes_host = planes

    def forward(self, x_bits, target, ws=None, with_pairs=True, path=dpa.PATH_AUTO):
        T = x_bits.shape[0]
        K = self.shape.top_k
        x = torch.from_numpy(x_bits.view(np.int16)).cuda()
        tg = torch.tensor([target], dtype=torch.float64, device="cuda")
        ws = dpa.new_workspace(self.desc, T) if ws is None else ws
        aux = {"topk_idx": torch.empty((T, K), dtype=torch.int32, device="cuda"),
               "topk_gate": torch.empty((T, K), dtype=torch.float64, device="cuda"),
               "k": torch.empty((T, K), dtype=torch.uint8, device="cuda"),
               "lambda": torch.empty(1, dtype=torch.float64, device="cuda"),
               "expert_path": path}
        if with_pairs:
            aux["pair_out"] = torch.empty((T, K, self.shape.hidden), dtype=torch.float32, device="cuda")
        y = dpa.moe_forward(self.layer, x, tg, ws, aux=aux)
        detail = dpa.device_error_detail(ws)
        st = dpa.device_status(ws)
        assert st == 0, (dpa.STATUS_NAMES.get(st, st), hex(detail[1]))
        out = {k: v.cpu().numpy() for k, v in aux.items() if k != "expert_path"}
        return bits_to_f64(y), out, ws


def check_forward(shape, x_bits, target, sample_pairs=None, token_subset=None, path=dpa.PATH_AUTO, pair_tol=1e-3):
    gl = GpuLayer.get(shape)
    y, aux, _ = gl.forward(x_bits, target, path=path)
    y_ref, ref = reference_layer(shape, x_bits, target, token_subset=token_subset)
    assert np.array_equal(aux["topk_idx"], ref["idx"])
    assert np.array_equal(aux["topk_gate"], ref["gates"])       # bit-identical fp64
    assert np.array_equal(aux["k"].astype(np.int64), ref["k"])
    assert aux["lambda"][0] == ref["lambda"]
    rows = np.arange(x_bits.shape[0]) if token_subset is None else np.asarray(token_subset)
    ok, worst = within_tol(y[rows], y_ref[rows], bf16_out=True)
    assert ok, f"output tolerance exceeded: worst err/bound = {worst}"
    if sample_pairs is not None:
        ref_o = pair_outputs(shape, x_bits, ref, sample_pairs)
        for (t, j), o in ref_o.items():
            ok, worst = within_tol(aux["pair_out"][t, j].astype(np.float64), o, pair_tol)
            assert ok, (t, j, worst)
    # the achieved average never exceeds the target
    assert aux["k"].astype(np.int64).sum() <= target * aux["k"].size
    return y, aux, ref


# ----------------------------------------------------------------------------- routing

@pytest.mark.parametrize("shape,T", [(W.TINY, 4), (W.QWEN3_B1, 1), (W.QWEN3_B64, 64), (W.DEEPSEEK_B16, 16),
                                     (W.QWEN3_B1, 37), (W.TINY, 3),
                                     # from 2 tokens on: tiled fp64 GEMM (ragged token tiles)
                                     (W.TINY, 200), (W.DEEPSEEK_B16, 130), (W.QWEN3_B64, 300)])
def test_route_bit_exact(shape, T):
    d = dpa.make_desc(shape)
    wr = W.router_weights(shape)
    x_bits = W.tokens(shape, T, step=11)
    ws = dpa.new_workspace(d, T)
    logits = torch.empty((T, shape.n_experts), dtype=torch.float64, device="cuda")
    idx, gate = dpa.route(d, torch.from_numpy(x_bits.view(np.int16)).cuda(),
                          torch.from_numpy(wr.view(np.int16)).cuda(), ws, logits=logits)
    assert dpa.device_status(ws) == 0
    ridx, rg, rl = O.route(x_bits, wr, shape.top_k, shape.norm_topk)
    assert np.array_equal(logits.cpu().numpy(), rl)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(gate.cpu().numpy(), rg)


@pytest.mark.parametrize("T", [4, 150])
def test_route_exact_path_for_wide_exponent_spread(T):
    # operands spread over ~200 binades, and large terms that cancel exactly, so the logit is
    # decided by tiny terms: the fp64 fast path cannot prove exactness and the kernel must
    # take the fixed-point path (per-logit kernel at 4 tokens, tiled kernel's fallback at 150)
    shape = W.with_sizes(W.TINY, name="tiny_spread")
    d = dpa.make_desc(shape)
    rng = np.random.default_rng(5)
    H, E = shape.hidden, shape.n_experts
    x = rng.standard_normal((T, H)).astype(np.float32)
    x[:, 0] = 2.0 ** 100
    x[:, 1] = -(2.0 ** 100)
    x[:, 2:10] *= np.float32(2.0 ** -100)
    w = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    w[:, 1] = w[:, 0]
    w[:, 10:20] *= np.float32(2.0 ** -60)
    xb, wb = W.f32_to_bf16_bits(x), W.f32_to_bf16_bits(w)
    ws = dpa.new_workspace(d, T)
    logits = torch.empty((T, E), dtype=torch.float64, device="cuda")
    idx, gate = dpa.route(d, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(wb.view(np.int16)).cuda(),
                          ws, logits=logits)
    assert dpa.device_status(ws) == 0
    ridx, rg, rl = O.route(xb, wb, shape.top_k, shape.norm_topk)
    assert np.array_equal(logits.cpu().numpy(), rl)
    assert np.array_equal(idx.cpu().numpy(), ridx) and np.array_equal(gate.cpu().numpy(), rg)


@pytest.mark.parametrize("case", ["tiny_elements", "block_scales"])
def test_route_tiled_slice_bounds(case):
    # The tiled router proves a logit exact by a whole-row bound or, failing that, by per-slice
    # bounds and a bound on the sum of the slice sums. tiny_elements: one element of 2^-30 per
    # token, so that the whole-row bound fails for ~1/6 of the logits, the per-slice bounds rescue
    # more than half of those and the rest is recomputed; block_scales: blocks of 64 inputs at
    # 2^-40, 1 and 2^40, so every slice is exact on its own and their sum never is.
    shape = W.with_sizes(W.TINY, name="tiny_slices")
    d = dpa.make_desc(shape)
    T, H, E = 64, shape.hidden, shape.n_experts
    rng = np.random.default_rng(17)
    x = rng.standard_normal((T, H)).astype(np.float32)
    w = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    if case == "tiny_elements":
        x[np.arange(T), rng.integers(0, H, T)] = np.float32(2.0 ** -30)
    else:
        for b in range(H // 64):
            x[:, 64 * b:64 * (b + 1)] *= np.float32(2.0 ** (40 * (b % 3 - 1)))
    xb, wb = W.f32_to_bf16_bits(x), W.f32_to_bf16_bits(w)
    ws = dpa.new_workspace(d, T)
    logits = torch.empty((T, E), dtype=torch.float64, device="cuda")
    idx, gate = dpa.route(d, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(wb.view(np.int16)).cuda(),
                          ws, logits=logits)
    assert dpa.device_status(ws) == 0
    ridx, rg, rl = O.route(xb, wb, shape.top_k, shape.norm_topk)
    assert np.array_equal(logits.cpu().numpy(), rl)
    assert np.array_equal(idx.cpu().numpy(), ridx) and np.array_equal(gate.cpu().numpy(), rg)


@pytest.mark.parametrize("E,K,T", [(64, 6, 1), (64, 6, 64), (256, 8, 1), (256, 8, 64)])
def test_route_ties_and_expert_counts(E, K, T):
    # Routers with repeated rows (equal logits: ties go to the lower expert id) at 64 experts,
    # where the top-k runs as warp extraction, and at 256 experts, where it runs as ranks (the
    # extraction covers at most 32 candidates); one token (per-logit kernel) and 64 (tiled).
    shape = W.with_sizes(W.QWEN3_B1, n_experts=E, top_k=K, name=f"route_e{E}")
    d = dpa.make_desc(shape)
    rng = np.random.default_rng(E * 100 + T)
    w = (rng.standard_normal((E, shape.hidden)) * 0.02).astype(np.float32)
    for dst in range(1, E, 3):   # every third row repeats an earlier one
        w[dst] = w[int(rng.integers(0, dst))]
    wb = W.f32_to_bf16_bits(w)
    xb = W.tokens(shape, T, step=21)
    ws = dpa.new_workspace(d, T)
    logits = torch.empty((T, E), dtype=torch.float64, device="cuda")
    idx, gate = dpa.route(d, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(wb.view(np.int16)).cuda(),
                          ws, logits=logits)
    assert dpa.device_status(ws) == 0
    ridx, rg, rl = O.route(xb, wb, K, shape.norm_topk)
    assert np.array_equal(logits.cpu().numpy(), rl)
    assert np.array_equal(idx.cpu().numpy(), ridx) and np.array_equal(gate.cpu().numpy(), rg)
    # the repeated rows do produce equal logits among the selected experts' rivals
    assert any(len(np.unique(rl[t])) < E for t in range(T))


# ----------------------------------------------------------------------------- allocation

def _alloc_inputs(seed, T, K, E, B, ties=False):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    g = -np.sort(-rng.dirichlet(np.ones(K), size=T), axis=1)
    if ties:
        g[:] = g[0]
        idx[:] = idx[0]
    base = rng.random(E) * 10 + 1
    r = np.stack([base * 4.0 ** (B - k) * (1 + 0.3 * rng.random(E)) for k in range(1, B + 1)], axis=1)
    return idx, g, r


@pytest.mark.parametrize("T,K,E,kmin,kmax,B,target,ties", [
    (4, 2, 8, 2, 4, 4, 3.0, False), (1, 8, 128, 2, 4, 4, 2.5, False), (64, 8, 128, 2, 4, 4, 2.0, False),
    (64, 8, 128, 2, 4, 4, 3.5, False), (64, 8, 128, 2, 4, 4, 4.0, False), (16, 6, 64, 1, 3, 3, 2.0, False),
    (2048, 8, 128, 2, 4, 4, 3.0, False), (7, 3, 16, 1, 4, 4, 2.75, False), (32, 8, 128, 2, 4, 4, 3.0, True),
    # mid-size batches (block-scale speculation and verification): edge of the range, four
    # plane counts, ties
    (256, 8, 128, 2, 4, 4, 2.5, False), (100, 8, 128, 1, 4, 4, 1.7, False), (64, 8, 128, 2, 4, 4, 3.0, True),
    (9, 8, 128, 2, 4, 4, 2.2, False),
    # up to 32 pairs (one warp): a single pair, the 32-pair edge, budgets at kmin and kmax,
    # duplicated pairs, three-plane BCQ-like ranges; 33 pairs falls back to the block kernel
    (1, 1, 8, 1, 4, 4, 1.0, False), (1, 1, 8, 1, 4, 4, 2.6, False), (4, 8, 128, 2, 4, 4, 2.0, False),
    (4, 8, 128, 2, 4, 4, 4.0, False), (4, 8, 128, 2, 4, 4, 3.3, False), (4, 8, 128, 2, 4, 4, 2.5, True),
    (5, 6, 64, 1, 3, 3, 2.0, False), (2, 8, 128, 2, 4, 4, 3.1, False), (11, 3, 16, 1, 4, 4, 2.4, False)])
def test_allocate_bit_exact(T, K, E, kmin, kmax, B, target, ties):
    shape = W.with_sizes(W.QWEN3_B1, n_experts=E, top_k=K, kmin=kmin, kmax=kmax, bits=B, name="alloc")
    d = dpa.make_desc(shape)
    idx, g, r = _alloc_inputs(T * 1000 + E, T, K, E, B, ties)
    rk, rlam = O.allocate(idx, g, r, kmin, kmax, target)
    ws = dpa.new_workspace(d, T)
    k, lam = dpa.allocate(d, torch.from_numpy(r).cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(g).cuda(),
                          torch.tensor([target], dtype=torch.float64, device="cuda"), ws)
    assert dpa.device_status(ws) == 0
    assert np.array_equal(k.cpu().numpy().astype(np.int64), rk)
    assert lam.item() == rlam


def test_allocate_invalid_target_sets_device_flag():
    shape = W.TINY
    d = dpa.make_desc(shape)
    idx, g, r = _alloc_inputs(1, 4, 2, 8, 4)
    ws = dpa.new_workspace(d, 4)
    k0 = torch.full((4, 2), 7, dtype=torch.uint8, device="cuda")
    for bad in (1.5, 4.5, float("nan")):
        st = dpa.lib().dpa_allocate(dpa.ctypes.byref(d), torch.from_numpy(r).cuda().data_ptr(),
                                    torch.from_numpy(idx).cuda().data_ptr(), torch.from_numpy(g).cuda().data_ptr(), 4,
                                    torch.tensor([bad], dtype=torch.float64, device="cuda").data_ptr(), k0.data_ptr(),
                                    None, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
        assert st == 0
        assert dpa.device_status(ws) == 6
        assert torch.all(k0 == 7)          # outputs untouched
    assert dpa.device_status(ws) == 0      # flag cleared


# ----------------------------------------------------------------------------- full layer

def test_forward_tiny():
    x = W.tokens(W.TINY)
    check_forward(W.TINY, x, 3.0, sample_pairs=[(t, j) for t in range(4) for j in range(2)])


@pytest.mark.parametrize("T", [1, 3, 8])
def test_forward_tiny_ragged_and_targets(T):
    x = W.tokens(W.TINY, T, step=T)
    for target in (2.0, 2.5, 4.0):
        check_forward(W.TINY, x, target)


def test_forward_qwen3_batch1():
    x = W.tokens(W.QWEN3_B1)
    check_forward(W.QWEN3_B1, x, 2.5, sample_pairs=[(0, j) for j in range(8)])


@pytest.mark.parametrize("target", [2.0, 2.5, 3.0, 3.5, 4.0])
def test_forward_qwen3_batch64_sampled(target):
    x = W.tokens(W.QWEN3_B64)
    check_forward(W.QWEN3_B64, x, target, token_subset=[0, 5, 31, 63],
                  sample_pairs=[(5, 0), (31, 7), (63, 3)])


def test_forward_deepseek_bcq_shared():
    x = W.tokens(W.DEEPSEEK_B16)
    check_forward(W.DEEPSEEK_B16, x, 2.0, token_subset=[0, 7, 15], sample_pairs=[(0, 0), (15, 5)])


def test_prefix_property_poisoned_planes():
    # at target = kmin every pair reads kmin planes: overwriting planes >= kmin of every
    # expert in device memory must not change a single output bit
    shape = W.TINY
    gl = GpuLayer.get(shape)
    x = W.tokens(shape, 4, step=3)
    y0, aux0, _ = gl.forward(x, float(shape.kmin))
    assert np.all(aux0["k"] == shape.kmin)
    s = dpa.encoded_sizes(gl.desc)
    saved = gl.layer.planes.clone()
    try:
        p = gl.layer.planes
        for e in range(shape.n_experts):
            for m in range(3):
                R = shape.hidden if m == 2 else shape.inter
                C = shape.inter if m == 2 else shape.hidden
                pb = R * C // 8
                start = e * s.planes_per_expert + s.planes_matrix_offset[m]
                p[start + shape.kmin * pb: start + shape.bits * pb] = 0xA5
        torch.cuda.synchronize()
        y1, aux1, _ = gl.forward(x, float(shape.kmin))
        assert np.array_equal(y0, y1)
    finally:
        gl.layer.planes.copy_(saved)


def _poison_unread(gl, idx, k, seed_byte=0xA5):
    """Overwrite, in device memory, every byte the forward must not read: planes >= kmax_e of
    each routed expert e (kmax_e = the largest k among its pairs; for binary-coded layers also
    those planes' alphas, with NaN), and all planes and scale data of experts nobody routed to
    (scales and zeros as NaN). Returns the saved copies."""
    shape = gl.shape
    s = dpa.encoded_sizes(gl.desc)
    saved = (gl.layer.planes.clone(), gl.layer.meta.clone())
    kmax_e = {}
    for e, kk in zip(idx.reshape(-1).tolist(), k.reshape(-1).tolist()):
        kmax_e[e] = max(kmax_e.get(e, 0), int(kk))
    p, mt = gl.layer.planes, gl.layer.meta
    H, I, G, B = shape.hidden, shape.inter, shape.group, shape.bits
    for e in range(shape.n_experts):
        km = kmax_e.get(e, 0)
        for m in range(3):
            R, C = (H, I) if m == 2 else (I, H)
            pb = R * C // 8
            start = e * s.planes_per_expert + s.planes_matrix_offset[m]
            p[start + km * pb: start + B * pb] = seed_byte
            mstart = e * s.meta_per_expert + s.meta_matrix_offset[m]
            if shape.fmt == W.FMT_BCQ:
                ab = R * (C // G) * 2          # one plane's alphas
                mt[mstart + km * ab: mstart + B * ab] = 0xFF
            elif km == 0:
                mt[mstart: mstart + R * (C // G) * 4] = 0xFF
    torch.cuda.synchronize()
    return saved


@pytest.mark.parametrize("shape,T,target", [(W.QWEN3_B64, 4, 2.5), (W.QWEN3_B64, 9, 3.0), (W.QWEN3_B1, 1, 2.5),
                                            (W.DEEPSEEK_B16, 16, 2.0)])
def test_prefix_property_mixed_k_poisoned(shape, T, target):
    # mixed plane counts: each routed expert reads only its first kmax_e planes (and, binary-coded,
    # their alphas); poisoning everything beyond, and every unrouted expert, changes no output bit
    gl = GpuLayer.get(shape)
    x = W.tokens(shape, T, step=41)
    y0, aux0, _ = gl.forward(x, target)
    assert len(np.unique(aux0["k"])) > 1
    saved = _poison_unread(gl, aux0["topk_idx"], aux0["k"])
    try:
        y1, aux1, _ = gl.forward(x, target)
        assert np.array_equal(aux1["k"], aux0["k"])
        assert np.array_equal(y0, y1)
        assert np.array_equal(aux0["pair_out"], aux1["pair_out"])
    finally:
        gl.layer.planes.copy_(saved[0])
        gl.layer.meta.copy_(saved[1])
        torch.cuda.synchronize()


def test_forward_activation_groups_spanning_many_binades():
    # the expert kernels hold each scale group of activations as 15-bit fixed point under the
    # group's largest exponent; groups spanning ~40 binades (magnitudes 2^-38 .. 2) lose only
    # digits far below the tolerance
    shape = W.TINY
    rng = np.random.default_rng(77)
    T, H = 6, shape.hidden
    mag = np.exp2(rng.integers(-38, 1, size=(T, H)).astype(np.float64))
    x = (mag * np.sign(rng.standard_normal((T, H))) * (1 + rng.random((T, H)))).astype(np.float32)
    xb = W.f32_to_bf16_bits(x)
    for target in (2.0, 3.0, 4.0):
        check_forward(shape, xb, target, sample_pairs=[(0, 0), (T - 1, 1)])


@pytest.mark.parametrize("fmt", [W.FMT_UNIFORM, W.FMT_BCQ])
def test_forward_wide_hidden_several_tiles_per_expert(fmt):
    # hidden 8192: the multi-token staging does not fit, so experts with many tokens run one
    # two-token tile per pass, several passes per work item (8 experts, top-2, 16 tokens)
    if fmt == W.FMT_UNIFORM:
        shape = W.with_sizes(W.TINY, name="wide_h8192_uniform", hidden=8192, inter=512, group=128, tokens=16,
                             seed=61)
        target = 3.0
    else:
        shape = W.with_sizes(W.TINY, name="wide_h8192_bcq", hidden=8192, inter=512, group=128, tokens=16, fmt=W.FMT_BCQ,
                             bits=3, kmin=1, kmax=3, norm_topk=0, seed=62)
        target = 2.0
    x = W.tokens(shape, 16, step=5)
    y, aux, ref = check_forward(shape, x, target, sample_pairs=[(0, 0), (15, 1), (7, 0)])
    counts = np.bincount(aux["topk_idx"].reshape(-1), minlength=shape.n_experts)
    assert counts.max() >= 3


def test_forward_deterministic_and_graph_capture():
    shape = W.TINY
    gl = GpuLayer.get(shape)
    x_bits = W.tokens(shape, 4, step=9)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    tg = torch.tensor([3.0], dtype=torch.float64, device="cuda")
    ws = dpa.new_workspace(gl.desc, 4)
    y_eager = dpa.moe_forward(gl.layer, x, tg, ws).clone()
    y_again = dpa.moe_forward(gl.layer, x, tg, ws).clone()
    assert torch.equal(y_eager, y_again)
    y_buf = torch.empty_like(y_eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dpa.moe_forward(gl.layer, x, tg, ws, y=y_buf, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        dpa.moe_forward(gl.layer, x, tg, ws, y=y_buf)
    for target in (3.0, 2.0, 4.0):
        tg.fill_(target)
        graph.replay()
        torch.cuda.synchronize()
        y_ref = dpa.moe_forward(gl.layer, x, tg, ws).clone()
        assert torch.equal(y_buf, y_ref)
    assert dpa.device_status(ws) == 0
