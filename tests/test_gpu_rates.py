"""Workload-profiled per-expert read rates (DuoRate abstract) through the C ABI against the
oracle: the prefill profile and the solved rate table are bit-identical, and decode steps that
read each expert at its table rate match the oracle within 2e-3 * (1 + |ref|)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from dynamic_any_precision_b200 import dpa, workloads as W  # noqa: E402
from oracle import dpa_oracle as O  # noqa: E402
from oracle_jobs import encode_experts, route_parallel  # noqa: E402
from test_gpu_parity import GpuLayer, bits_to_f64, within_tol  # noqa: E402

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _scalar(v):
    return torch.tensor([v], dtype=torch.float64, device="cuda")


@pytest.mark.parametrize("shape,T", [(W.TINY, 37), (W.QWEN3_B64, 300)])
def test_prefill_profile_bit_exact(shape, T):
    d = dpa.make_desc(shape)
    x = W.tokens(shape, T, step=71)
    rng = np.random.default_rng(T)
    idx = np.stack([rng.choice(shape.n_experts, shape.top_k, replace=False) for _ in range(T)]).astype(np.int32)
    ws = dpa.new_workspace(d, 1)
    m, c = dpa.profile_prefill(d, _dev(x.view(np.int16)), _dev(idx), ws)
    assert dpa.device_status(ws) == 0
    m_ref, c_ref = O.prefill_profile(x, idx, shape.n_experts)
    assert np.array_equal(m.cpu().numpy(), m_ref)
    assert np.array_equal(c.cpu().numpy().astype(np.int64), c_ref)


@pytest.mark.parametrize("E,B,kmin,kmax,H,target,seed", [(8, 4, 2, 4, 256, 3.0, 0), (128, 4, 2, 4, 2048, 2.5, 1),
                                                         (128, 4, 2, 4, 2048, 3.3, 2), (64, 3, 1, 3, 2048, 2.0, 3),
                                                         (128, 4, 2, 4, 2048, 4.0, 4), (16, 4, 1, 4, 512, 1.7, 5)])
def test_solve_expert_rates_bit_exact(E, B, kmin, kmax, H, target, seed):
    # a seeded synthetic distortion tensor (decreasing ~4x per plane) and profile
    shape = W.with_sizes(W.QWEN3_B1, n_experts=E, bits=B, kmin=kmin, kmax=kmax, hidden=H, name="rates")
    d = dpa.make_desc(shape)
    rng = np.random.default_rng(seed)
    base = rng.random((E, 1)) * 5 + 0.5
    Td = np.stack([base * 4.0 ** (B - k) * (1 + 0.2 * rng.random((E, H))) for k in range(1, B + 1)], axis=1)
    m = rng.random(H) + 0.1
    counts = rng.integers(0, 12, size=E).astype(np.int32)
    ws = dpa.new_workspace(d, 1)
    kt, lam = dpa.solve_expert_rates(d, _dev(Td), _dev(m), _dev(counts), _scalar(target), ws)
    assert dpa.device_status(ws) == 0
    k_ref, lam_ref, _ = O.solve_expert_rates(Td, m, counts.astype(np.int64), kmin, kmax, target)
    assert np.array_equal(kt.cpu().numpy().astype(np.int64), k_ref)
    assert lam.item() == lam_ref


def test_solve_expert_rates_rejects_out_of_range_target():
    d = dpa.make_desc(W.TINY)
    ws = dpa.new_workspace(d, 1)
    kt = torch.full((8,), 9, dtype=torch.uint8, device="cuda")
    Td = _dev(np.ones((8, 4, 256)))
    st = dpa.lib().dpa_solve_expert_rates(dpa.ctypes.byref(d), Td.data_ptr(), _dev(np.ones(256)).data_ptr(),
                                          _dev(np.ones(8, np.int32)).data_ptr(), _scalar(1.0).data_ptr(),
                                          kt.data_ptr(), None, ws.data_ptr(), ws.numel(),
                                          torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert dpa.device_status(ws) == 6 and torch.all(kt == 9)


@pytest.mark.parametrize("target", [2.5, 3.0])
def test_duorate_end_to_end_tiny(target):
    # offline: encode + distortion tensor; online: route a prefill, profile it, solve the table;
    # decode: every pair reads its expert's rate. Each step is compared with the oracle's.
    shape = W.TINY
    gl = GpuLayer.get(shape)
    d = gl.desc
    g, u, dn = W.all_expert_weights(shape)
    planes, meta, _ = dpa.encode(d, g, u, dn)
    Td = dpa.distortion_tensor(d, g, u, planes, meta)
    experts = encode_experts(shape, range(shape.n_experts))
    Td_ref = np.stack([O.distortion_tensor(experts[e], shape.fmt, shape.bits, shape.group, g[e], u[e])
                       for e in range(shape.n_experts)])
    assert np.array_equal(Td, Td_ref)
    xp = W.tokens(shape, 64, step=500)
    wr = W.router_weights(shape)
    ws = dpa.new_workspace(d, 64)
    idx, _ = dpa.route(d, _dev(xp.view(np.int16)), _dev(wr.view(np.int16)), ws)
    m, c = dpa.profile_prefill(d, _dev(xp.view(np.int16)), idx, ws)
    kt, lam = dpa.solve_expert_rates(d, _dev(Td), m, c, _scalar(target), ws)
    assert dpa.device_status(ws) == 0
    idx_ref, _, _ = O.route(xp, wr, shape.top_k, shape.norm_topk)
    m_ref, c_ref = O.prefill_profile(xp, idx_ref, shape.n_experts)
    k_ref, lam_ref, _ = O.solve_expert_rates(Td_ref, m_ref, c_ref, shape.kmin, shape.kmax, target)
    assert np.array_equal(kt.cpu().numpy().astype(np.int64), k_ref) and lam.item() == lam_ref
    # decode with the table
    xd = W.tokens(shape, 6, step=501)
    aux = {"topk_idx": torch.empty((6, 2), dtype=torch.int32, device="cuda"),
           "k": torch.empty((6, 2), dtype=torch.uint8, device="cuda"),
           "alloc_policy": dpa.ALLOC_EXPERT_TABLE, "expert_k": kt}
    y = dpa.moe_forward(gl.layer, _dev(xd.view(np.int16)), _scalar(target), ws, aux=aux)
    assert dpa.device_status(ws) == 0
    y_ref, ref = O.moe_forward(xd, wr, experts, shape, target, policy=O.ALLOC_EXPERT_TABLE, expert_k=k_ref)
    assert np.array_equal(aux["k"].cpu().numpy().astype(np.int64), ref["k"])
    ok, worst = within_tol(bits_to_f64(y), y_ref, bf16_out=True)
    assert ok, worst


def test_expert_table_forward_qwen3_batch64():
    shape = W.QWEN3_B64
    gl = GpuLayer.get(shape)
    rng = np.random.default_rng(9)
    table = rng.integers(shape.kmin, shape.kmax + 1, size=shape.n_experts).astype(np.uint8)
    x = W.tokens(shape, 64, step=502)
    ws = dpa.new_workspace(gl.desc, 64)
    aux = {"topk_idx": torch.empty((64, 8), dtype=torch.int32, device="cuda"),
           "k": torch.empty((64, 8), dtype=torch.uint8, device="cuda"),
           "alloc_policy": dpa.ALLOC_EXPERT_TABLE, "expert_k": _dev(table)}
    y = dpa.moe_forward(gl.layer, _dev(x.view(np.int16)), _scalar(3.0), ws, aux=aux)
    assert dpa.device_status(ws) == 0
    wr = W.router_weights(shape)
    idx, g, lg = route_parallel(shape, x)
    experts = encode_experts(shape, np.unique(idx[[0, 33, 63]]))
    y_ref, ref = O.moe_forward(x, wr, experts, shape, 3.0, logits=lg, policy=O.ALLOC_EXPERT_TABLE,
                               expert_k=table.astype(np.int64), token_subset=[0, 33, 63])
    assert np.array_equal(aux["k"].cpu().numpy().astype(np.int64), table.astype(np.int64)[idx])
    ok, worst = within_tol(bits_to_f64(y)[[0, 33, 63]], y_ref[[0, 33, 63]], bf16_out=True)
    assert ok, worst
