"""Allocation policies other than the Lagrangian, through the C ABI against the fp64 oracle:
the uniform control (DPA-MoE abstract: uniform chunk allocation at matched budgets) and the
score-threshold policy with its calibration (MatMoE review, "Core Contribution"). Plane counts
and thresholds are bit-identical; layer outputs within 2e-3 * (1 + |ref|)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from dynamic_any_precision_b200 import dpa, workloads as W  # noqa: E402
from oracle import dpa_oracle as O  # noqa: E402
from oracle_jobs import encode_experts, route_parallel  # noqa: E402
from test_gpu_parity import GpuLayer, within_tol, bits_to_f64  # noqa: E402

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _scalar(v):
    return torch.tensor([v], dtype=torch.float64, device="cuda")


def _pairs(seed, T, K, E):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    g = -np.sort(-rng.dirichlet(np.ones(K), size=T), axis=1)
    return idx, g


@pytest.mark.parametrize("T,K,E,kmin,kmax,B,target", [
    (4, 2, 8, 2, 4, 4, 3.0), (1, 8, 128, 2, 4, 4, 2.5), (64, 8, 128, 2, 4, 4, 3.3), (16, 6, 64, 1, 3, 3, 1.9),
    (7, 3, 16, 1, 4, 4, 2.75), (2048, 8, 128, 2, 4, 4, 3.1), (3000, 8, 128, 2, 4, 4, 2.0)])
def test_allocate_uniform_bit_exact(T, K, E, kmin, kmax, B, target):
    shape = W.with_sizes(W.QWEN3_B1, n_experts=E, top_k=K, kmin=kmin, kmax=kmax, bits=B, name="alloc_u")
    d = dpa.make_desc(shape)
    idx, g = _pairs(T + E, T, K, E)
    ws = dpa.new_workspace(d, T)
    r = np.ones((E, B))
    k, lam = dpa.allocate(d, _dev(r), _dev(idx), _dev(g), _scalar(target), ws, policy=dpa.ALLOC_UNIFORM)
    assert dpa.device_status(ws) == 0
    want = O.allocate_uniform(T * K, kmin, kmax, target).reshape(T, K)
    assert np.array_equal(k.cpu().numpy().astype(np.int64), want)
    assert lam.item() == 0.0


@pytest.mark.parametrize("n,kmin,kmax,target,seed", [(512, 2, 4, 3.0, 0), (96, 1, 3, 2.0, 1), (16384, 2, 4, 2.5, 2),
                                                     (8, 2, 4, 4.0, 3), (8, 2, 4, 2.0, 4), (777, 2, 3, 2.4, 5)])
def test_calibrate_threshold_bit_exact(n, kmin, kmax, target, seed):
    shape = W.with_sizes(W.QWEN3_B1, kmin=kmin, kmax=kmax, name="calib")
    d = dpa.make_desc(shape)
    rng = np.random.default_rng(seed)
    scores = rng.dirichlet(np.ones(8), size=(n + 7) // 8).reshape(-1)[:n].copy()
    scores[: n // 10] = scores[0]            # ties
    ws = dpa.new_workspace(d, 1)
    tau = dpa.calibrate_threshold(d, _dev(scores), _scalar(target), ws)
    assert dpa.device_status(ws) == 0
    assert tau.item() == O.calibrate_threshold(scores, kmin, kmax, target)


def test_calibrate_threshold_on_routed_calibration_batch_and_allocate():
    # the calibration distribution is the gates of a calibration batch routed by the layer's own
    # router (routed by the oracle here); the threshold then drives a live batch's plane counts
    shape = W.QWEN3_B64
    d = dpa.make_desc(shape)
    xc = W.tokens(shape, 256, step=900)
    _, g_cal, _ = route_parallel(shape, xc)
    ws = dpa.new_workspace(d, 64)
    for target in (2.5, 3.0, 3.5):
        tau = dpa.calibrate_threshold(d, _dev(g_cal), _scalar(target), ws)
        assert dpa.device_status(ws) == 0
        tau_ref = O.calibrate_threshold(g_cal, shape.kmin, shape.kmax, target)
        assert tau.item() == tau_ref
        idx, g = _pairs(int(target * 10), 64, 8, 128)
        k, lam = dpa.allocate(d, None, _dev(idx), _dev(g), None, ws, policy=dpa.ALLOC_THRESHOLD, threshold=tau)
        assert dpa.device_status(ws) == 0
        assert np.array_equal(k.cpu().numpy().astype(np.int64), O.allocate_threshold(g, tau_ref, 2, 4))
        assert lam.item() == tau_ref


def test_invalid_policy_inputs():
    d = dpa.make_desc(W.TINY)
    idx, g = _pairs(1, 4, 2, 8)
    ws = dpa.new_workspace(d, 4)
    k0 = torch.full((4, 2), 7, dtype=torch.uint8, device="cuda")
    L = dpa.lib()
    args = (dpa.ctypes.byref(d),)
    # unknown policy, and a threshold policy without a threshold: rejected on the host
    for pol, thr in ((4, None), (dpa.ALLOC_THRESHOLD, None), (dpa.ALLOC_EXPERT_TABLE, None)):
        st = L.dpa_allocate_ex(*args, pol, None, _dev(idx).data_ptr(), _dev(g).data_ptr(), 4,
                               _scalar(3.0).data_ptr(), thr, None, k0.data_ptr(), None, ws.data_ptr(), ws.numel(),
                               torch.cuda.current_stream().cuda_stream)
        assert st == 1
    # a NaN threshold and an out-of-range calibration target: device flag, outputs untouched
    bad = _scalar(float("nan"))
    st = L.dpa_allocate_ex(*args, dpa.ALLOC_THRESHOLD, None, _dev(idx).data_ptr(), _dev(g).data_ptr(), 4, None,
                           bad.data_ptr(), None, k0.data_ptr(), None, ws.data_ptr(), ws.numel(),
                           torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert dpa.device_status(ws) == 6 and torch.all(k0 == 7)
    tau = _scalar(-5.0)
    gd = _dev(g)
    st = L.dpa_calibrate_threshold(*args, gd.data_ptr(), gd.numel(), _scalar(4.5).data_ptr(), tau.data_ptr(),
                                   ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert dpa.device_status(ws) == 6
    assert tau.item() == -5.0


def _forward_policy(shape, x_bits, target, policy, threshold=None, token_subset=None):
    gl = GpuLayer.get(shape)
    T, K = x_bits.shape[0], shape.top_k
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    ws = dpa.new_workspace(gl.desc, T)
    aux = {"topk_idx": torch.empty((T, K), dtype=torch.int32, device="cuda"),
           "topk_gate": torch.empty((T, K), dtype=torch.float64, device="cuda"),
           "k": torch.empty((T, K), dtype=torch.uint8, device="cuda"),
           "lambda": torch.empty(1, dtype=torch.float64, device="cuda"),
           "alloc_policy": policy, "threshold": None if threshold is None else _scalar(threshold)}
    y = dpa.moe_forward(gl.layer, x, _scalar(target), ws, aux=aux)
    assert dpa.device_status(ws) == 0
    wr = W.router_weights(shape)
    idx, g, lg = O.route(x_bits, wr, K, shape.norm_topk)
    experts = encode_experts(shape, np.unique(idx))
    y_ref, ref = O.moe_forward(x_bits, wr, experts, shape, target, logits=lg, policy=policy, threshold=threshold,
                               token_subset=token_subset)
    assert np.array_equal(aux["topk_idx"].cpu().numpy(), ref["idx"])
    assert np.array_equal(aux["k"].cpu().numpy().astype(np.int64), ref["k"])
    assert aux["lambda"].item() == ref["lambda"]
    rows = np.arange(T) if token_subset is None else np.asarray(token_subset)
    ok, worst = within_tol(bits_to_f64(y)[rows], y_ref[rows], bf16_out=True)
    assert ok, worst
    return ref


@pytest.mark.parametrize("target", [2.5, 3.0])
def test_forward_uniform_policy(target):
    ref = _forward_policy(W.TINY, W.tokens(W.TINY, 8, step=4), target, dpa.ALLOC_UNIFORM)
    assert ref["k"].sum() == int(target * 16)
    _forward_policy(W.QWEN3_B64, W.tokens(W.QWEN3_B64, 64, step=5), target, dpa.ALLOC_UNIFORM,
                    token_subset=[0, 21, 63])


def test_forward_threshold_policy():
    shape = W.QWEN3_B64
    _, g_cal, _ = route_parallel(shape, W.tokens(shape, 128, step=901))
    tau = O.calibrate_threshold(g_cal, shape.kmin, shape.kmax, 3.0)
    ref = _forward_policy(shape, W.tokens(shape, 64, step=6), 3.0, dpa.ALLOC_THRESHOLD, threshold=tau,
                          token_subset=[1, 40])
    assert set(np.unique(ref["k"]).tolist()) == {2, 4}
    _forward_policy(W.TINY, W.tokens(W.TINY, 6, step=7), 3.0, dpa.ALLOC_THRESHOLD, threshold=0.55)
