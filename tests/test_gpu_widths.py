"""Per-expert stored widths on the device (MatMoE, review "Core Contribution": each expert keeps
a solved maximum bit-width): a compact layer of each expert's plane prefix runs the forward with
every pair reading at most its expert's width. Decisions are bit-identical to the oracle's
(capped allocation), outputs within 2e-3 (1 + |ref|), and the compact layer's outputs are
bit-identical to the full layer's for the same plane counts."""
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


def _compact(gl, widths):
    shape = gl.shape
    d = gl.desc
    cp, cm, off = dpa.compact_layer(d, gl.planes_host, gl.layer.meta.cpu().numpy(), widths)
    return dpa.DeviceLayer(d, _dev(cp), _dev(cm), gl.layer.rtable, gl.layer.w_router, gl.layer.shared,
                           widths=_dev(widths.astype(np.uint8)), offsets=_dev(off.view(np.int64)))


def _widths(shape, gl, avg):
    # importance: routing mass of a synthetic calibration batch routed by the oracle
    xc = W.tokens(shape, 32, step=900)
    idx, g, _ = route_parallel(shape, xc)
    imp = O.routing_mass(idx, g, shape.n_experts)
    r = gl.layer.rtable.cpu().numpy()
    budget = int(avg * shape.n_experts)
    w = dpa.solve_stored_widths(gl.desc, imp, r, budget)
    assert np.array_equal(w.astype(np.int64), O.solve_stored_widths(imp, r, shape.kmin, shape.kmax, budget))
    return w


@pytest.mark.parametrize("shape,T,target,avg", [(W.TINY, 6, 3.0, 2.6), (W.QWEN3_B64, 64, 3.0, 3.1),
                                                (W.DEEPSEEK_B16, 16, 2.0, 2.2)])
def test_compact_layer_forward_matches_oracle(shape, T, target, avg):
    gl = GpuLayer.get(shape)
    widths = _widths(shape, gl, avg)
    layer = _compact(gl, widths)
    x = W.tokens(shape, T, step=901)
    K = shape.top_k
    ws = dpa.new_workspace(gl.desc, T)
    aux = {"topk_idx": torch.empty((T, K), dtype=torch.int32, device="cuda"),
           "k": torch.empty((T, K), dtype=torch.uint8, device="cuda")}
    y = dpa.moe_forward(layer, _dev(x.view(np.int16)), torch.tensor([target], dtype=torch.float64, device="cuda"),
                        ws, aux=aux)
    assert dpa.device_status(ws) == 0
    k = aux["k"].cpu().numpy().astype(np.int64)
    idx = aux["topk_idx"].cpu().numpy()
    assert np.all(k <= widths.astype(np.int64)[idx])
    sub = list(range(T)) if T <= 8 else [0, T // 2, T - 1]
    _, _, lg = route_parallel(shape, x)
    experts = encode_experts(shape, np.unique(idx[sub]))
    r_table = gl.layer.rtable.cpu().numpy()
    shared = W.shared_weights_bf16(shape) if shape.n_shared else None
    y_ref, ref = O.moe_forward(x, W.router_weights(shape), experts, shape, target, shared=shared, r_table=r_table,
                               logits=lg, token_subset=sub, widths=widths.astype(np.int64))
    assert np.array_equal(k, ref["k"])
    ok, worst = within_tol(bits_to_f64(y)[sub], y_ref[sub], bf16_out=True)
    assert ok, worst


def test_compact_layer_reads_the_same_planes_as_the_full_layer():
    # the expert-rate table policy with the widths as the table: every pair reads exactly its
    # expert's width from either layout, so the outputs must agree bit for bit
    shape = W.QWEN3_B64
    gl = GpuLayer.get(shape)
    rng = np.random.default_rng(7)
    widths = rng.integers(shape.kmin, shape.kmax + 1, size=shape.n_experts).astype(np.uint8)
    layer = _compact(gl, widths)
    x = _dev(W.tokens(shape, 64, step=902).view(np.int16))
    tg = torch.tensor([3.0], dtype=torch.float64, device="cuda")
    outs = []
    for lay in (gl.layer, layer):
        ws = dpa.new_workspace(gl.desc, 64)
        aux = {"alloc_policy": dpa.ALLOC_EXPERT_TABLE, "expert_k": _dev(widths)}
        outs.append(dpa.moe_forward(lay, x, tg, ws, aux=aux).clone())
        assert dpa.device_status(ws) == 0
    assert torch.equal(outs[0], outs[1])


def test_invalid_widths_set_the_device_flag_and_tc_path_is_refused():
    shape = W.TINY
    gl = GpuLayer.get(shape)
    widths = np.full(shape.n_experts, 3, np.uint8)
    layer = _compact(gl, widths)
    bad = _dev(np.full(shape.n_experts, 7, np.uint8))
    lay_bad = dpa.DeviceLayer(gl.desc, layer.planes, layer.meta, layer.rtable, layer.w_router, None,
                              widths=bad, offsets=layer.offsets)
    x = _dev(W.tokens(shape, 4, step=903).view(np.int16))
    tg = torch.tensor([3.0], dtype=torch.float64, device="cuda")
    ws = dpa.new_workspace(gl.desc, 4)
    dpa.moe_forward(lay_bad, x, tg, ws)
    assert dpa.device_status(ws) == 6
    with pytest.raises(dpa.DpaError, match="UNSUPPORTED"):
        dpa.moe_forward(layer, x, tg, ws, aux={"expert_path": dpa.PATH_TC})
