"""Stack glue (residual add + RMSNorm between layers) against the fp64 oracle, and a short
stack of layers run through the C ABI against the oracle's own stack from the same seeded
input (no value from the CUDA path enters the oracle)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from dynamic_any_precision_b200 import dpa, workloads as W  # noqa: E402
from oracle import dpa_oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu


def _half_ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 1e-300)))
    return np.ldexp(1.0, (e - 8).astype(int))


@pytest.mark.parametrize("T,H", [(1, 2048), (7, 256), (32, 2048)])
def test_residual_rmsnorm_matches_oracle(T, H):
    rng = np.random.default_rng(T * 100 + H)
    h0 = (rng.standard_normal((T, H)) * 3).astype(np.float32)
    y = W.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32) * 0.2)
    h = torch.from_numpy(h0.copy()).cuda()
    x = torch.empty((T, H), dtype=torch.int16, device="cuda")
    dpa.residual_rmsnorm(h, x, torch.from_numpy(y.view(np.int16)).cuda())
    torch.cuda.synchronize()
    h_ref = h0.astype(np.float64) + O.bf16_bits_to_f64(y)
    x_ref = O.rmsnorm(h_ref)
    np.testing.assert_allclose(h.cpu().numpy(), h_ref, rtol=1e-7, atol=1e-7)
    xg = O.bf16_bits_to_f64(x.cpu().numpy().view(np.uint16))
    # the GPU value is a bf16 rounding of an fp32 computation: within half a bf16 ulp of the
    # exact value, plus the fp32 error of the norm
    assert np.all(np.abs(xg - x_ref) <= _half_ulp_bf16(x_ref) * 1.0001 + 2e-6 * np.abs(x_ref) + 1e-30)
    # without y: pure normalisation, h untouched
    h2 = torch.from_numpy(h0.copy()).cuda()
    dpa.residual_rmsnorm(h2, x)
    torch.cuda.synchronize()
    assert np.array_equal(h2.cpu().numpy(), h0)
    xg = O.bf16_bits_to_f64(x.cpu().numpy().view(np.uint16))
    x_ref = O.rmsnorm(h0.astype(np.float64))
    assert np.all(np.abs(xg - x_ref) <= _half_ulp_bf16(x_ref) * 1.0001 + 2e-6 * np.abs(x_ref) + 1e-30)


def _oracle_stack(shape, n_layers, tokens_bits):
    """The oracle's own stack from the same seeded tokens: per layer x = bf16(RMSNorm(h)),
    y = bf16(MoE(x)) (the layer output format), h += y."""
    from oracle_jobs import encode_experts
    h = O.bf16_bits_to_f64(tokens_bits)
    xs, decisions = [], []
    for layer in range(n_layers):
        seed = W.layer_seed(shape, layer)
        x_bits = O.f64_to_bf16_bits(O.rmsnorm(h))
        wr = W.router_weights(shape, seed)
        idx, g, lg = O.route(x_bits, wr, shape.top_k, shape.norm_topk)
        experts = encode_experts(shape, np.unique(idx), seed)
        r = np.full((shape.n_experts, shape.bits), np.nan)
        for e, enc in experts.items():
            r[e] = enc["r"]
        y, aux = O.moe_forward(x_bits, wr, experts, shape, shape.targets[0], r_table=r, logits=lg)
        xs.append(x_bits)
        decisions.append(aux)
        h = h + O.bf16_bits_to_f64(O.f64_to_bf16_bits(y))
    return h, xs, decisions


@pytest.mark.parametrize("shape,n_layers,T", [(W.with_sizes(W.TINY, layers=3, name="tiny_stack"), 3, 4),
                                              (W.with_sizes(W.QWEN3_STACK, tokens=4), 2, 4)])
def test_stack_matches_oracle_stack(shape, n_layers, T):
    from dynamic_any_precision_b200.stack import DeviceStack, initial_stream
    stack = DeviceStack(shape, n_layers=n_layers)
    bufs = stack.buffers(T)
    tok = W.tokens(shape, T, step=77)
    h = torch.from_numpy(W.bf16_bits_to_f32(tok).astype(np.float32)).cuda()
    K = shape.top_k
    auxs = [{"topk_idx": torch.empty((T, K), dtype=torch.int32, device="cuda"),
             "topk_gate": torch.empty((T, K), dtype=torch.float64, device="cuda"),
             "k": torch.empty((T, K), dtype=torch.uint8, device="cuda"),
             "lambda": torch.empty(1, dtype=torch.float64, device="cuda")} for _ in range(n_layers)]
    # record every layer's input x on the GPU: run the layers one at a time
    target = torch.tensor([shape.targets[0]], dtype=torch.float64, device="cuda")
    x, y, ws = bufs["x"], bufs["y"], bufs["ws"]
    gpu_xs = []
    dpa.residual_rmsnorm(h, x)
    for layer in range(n_layers):
        gpu_xs.append(x.cpu().numpy().view(np.uint16).copy())
        dpa.moe_forward(stack.layers[layer], x, target, ws, y=y, aux=auxs[layer])
        dpa.residual_rmsnorm(h, x, y)
    torch.cuda.synchronize()
    assert dpa.device_status(ws) == 0
    h_ref, ref_xs, ref_dec = _oracle_stack(shape, n_layers, tok)
    same_inputs = True
    for layer in range(n_layers):
        if not np.array_equal(gpu_xs[layer], ref_xs[layer]):
            # a bf16 rounding boundary separated the two sides' layer inputs: from here on the
            # decisions may legitimately differ; the inputs must still agree to one bf16 step
            d = np.abs(O.bf16_bits_to_f64(gpu_xs[layer]) - O.bf16_bits_to_f64(ref_xs[layer]))
            assert np.all(d <= 2.0 ** -7 * np.maximum(1.0, np.abs(O.bf16_bits_to_f64(ref_xs[layer]))))
            same_inputs = False
            break
        a = {k: v.cpu().numpy() for k, v in auxs[layer].items()}
        assert np.array_equal(a["topk_idx"], ref_dec[layer]["idx"])
        assert np.array_equal(a["topk_gate"], ref_dec[layer]["gates"])
        assert np.array_equal(a["k"].astype(np.int64), ref_dec[layer]["k"])
        assert a["lambda"][0] == ref_dec[layer]["lambda"]
    if same_inputs:
        hg = h.cpu().numpy().astype(np.float64)
        err = np.abs(hg - h_ref) / (2e-3 * (1.0 + np.abs(h_ref)))
        assert float(err.max()) <= 1.0, float(err.max())
