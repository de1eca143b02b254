"""Stack glue (residual add + RMSNorm between layers) against the fp64 oracle, and stacks of
layers run through the C ABI, checked layer by layer:
  - on the oracle's own chain: the oracle runs the stack from the seeded tokens and each GPU
    layer is fed the oracle's input of that layer (short stacks, every layer);
  - teacher-forced: the GPU runs the stack and the oracle recomputes each checked layer from the
    input the GPU stack gave that layer, so a rounding difference in an earlier layer never
    stops the comparison (short stacks every layer; the 48-layer stack on sampled layers)."""
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


def _run_stack_recording(stack, h, target, T, n_layers):
    """Run the layers one at a time on the GPU, recording each layer's input x, output y and
    decisions (the layers see exactly what the stack's forward gives them)."""
    K = stack.shape.top_k
    bufs = stack.buffers(T)
    x, y, ws = bufs["x"], bufs["y"], bufs["ws"]
    rec = []
    dpa.residual_rmsnorm(h, x)
    for layer in range(n_layers):
        aux = {"topk_idx": torch.empty((T, K), dtype=torch.int32, device="cuda"),
               "topk_gate": torch.empty((T, K), dtype=torch.float64, device="cuda"),
               "k": torch.empty((T, K), dtype=torch.uint8, device="cuda"),
               "lambda": torch.empty(1, dtype=torch.float64, device="cuda")}
        xin = x.clone()
        dpa.moe_forward(stack.layers[layer], x, target, ws, y=y, aux=aux)
        rec.append({"x": xin, "y": y.clone(), **aux})
        dpa.residual_rmsnorm(h, x, y)
    torch.cuda.synchronize()
    assert dpa.device_status(ws) == 0
    return [{k: v.cpu().numpy() for k, v in r.items()} for r in rec]


def _check_layer_teacher_forced(shape, layer, r, target, token_subset):
    """The oracle runs layer `layer` on the GPU's own input of that layer: routing and allocation
    of every token bit-identical, outputs of the subset within 2e-3 (GPU y is bf16)."""
    from oracle_jobs import reference_layer_parallel
    seed = W.layer_seed(shape, layer)
    x_bits = r["x"].view(np.uint16)
    y_ref, ref = reference_layer_parallel(shape, x_bits, target, token_subset, seed=seed)
    assert np.array_equal(r["topk_idx"], ref["idx"]), layer
    assert np.array_equal(r["topk_gate"], ref["gates"]), layer
    assert np.array_equal(r["k"].astype(np.int64), ref["k"]), layer
    assert r["lambda"][0] == ref["lambda"], layer
    from test_gpu_parity import within_tol
    yg = O.bf16_bits_to_f64(r["y"].view(np.uint16))
    ok, worst = within_tol(yg[token_subset], y_ref[token_subset], bf16_out=True)
    assert ok, (layer, worst)


@pytest.mark.parametrize("shape,n_layers,T", [(W.with_sizes(W.TINY, layers=3, name="tiny_stack"), 3, 4),
                                              (W.with_sizes(W.QWEN3_STACK, tokens=4), 2, 4)])
def test_stack_teacher_forced_every_layer(shape, n_layers, T):
    # every layer is checked on the input the GPU stack actually gave it (teacher forcing), so a
    # rounding difference in an earlier layer never stops the comparison
    from dynamic_any_precision_b200.stack import DeviceStack
    stack = DeviceStack(shape, n_layers=n_layers)
    tok = W.tokens(shape, T, step=77)
    h = torch.from_numpy(W.bf16_bits_to_f32(tok).astype(np.float32)).cuda()
    target = shape.targets[0]
    rec = _run_stack_recording(stack, h, torch.tensor([target], dtype=torch.float64, device="cuda"), T, n_layers)
    for layer in range(n_layers):
        _check_layer_teacher_forced(shape, layer, rec[layer], target, list(range(T)))
    # the residual stream is the running sum of the layer outputs
    h_ref = W.bf16_bits_to_f32(tok).astype(np.float64)
    for r in rec:
        h_ref = h_ref + O.bf16_bits_to_f64(r["y"].view(np.uint16))
    np.testing.assert_allclose(h.cpu().numpy().astype(np.float64), h_ref, rtol=1e-6, atol=1e-6)


def _oracle_chain(shape, n_layers, tokens_bits):
    """The oracle's own stack from the seeded tokens: per layer x = bf16(RMSNorm(h)),
    y = MoE(x) rounded to bf16 (the layer output format), h += y. Returns every layer's input,
    output and decisions."""
    from oracle_jobs import encode_experts
    h = O.bf16_bits_to_f64(tokens_bits)
    out = []
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
        out.append({"x": x_bits, "y": y, **aux})
        h = h + O.bf16_bits_to_f64(O.f64_to_bf16_bits(y))
    return out


@pytest.mark.parametrize("shape,n_layers,T", [(W.with_sizes(W.TINY, layers=3, name="tiny_stack"), 3, 4),
                                              (W.with_sizes(W.QWEN3_STACK, tokens=4), 2, 4)])
def test_stack_layers_on_the_oracle_chain(shape, n_layers, T):
    # the other direction: the oracle runs the whole stack from the seeded tokens, and each GPU
    # layer is fed the oracle's input of that layer (so no oracle input comes from the GPU);
    # every layer's decisions are bit-identical and its output within 2e-3
    from dynamic_any_precision_b200.stack import DeviceStack
    stack = DeviceStack(shape, n_layers=n_layers)
    chain = _oracle_chain(shape, n_layers, W.tokens(shape, T, step=78))
    K = shape.top_k
    ws = dpa.new_workspace(stack.desc, T)
    tg = torch.tensor([shape.targets[0]], dtype=torch.float64, device="cuda")
    for layer, ref in enumerate(chain):
        aux = {"topk_idx": torch.empty((T, K), dtype=torch.int32, device="cuda"),
               "topk_gate": torch.empty((T, K), dtype=torch.float64, device="cuda"),
               "k": torch.empty((T, K), dtype=torch.uint8, device="cuda"),
               "lambda": torch.empty(1, dtype=torch.float64, device="cuda")}
        x = torch.from_numpy(ref["x"].view(np.int16)).cuda()
        y = dpa.moe_forward(stack.layers[layer], x, tg, ws, aux=aux)
        assert dpa.device_status(ws) == 0
        assert np.array_equal(aux["topk_idx"].cpu().numpy(), ref["idx"]), layer
        assert np.array_equal(aux["topk_gate"].cpu().numpy(), ref["gates"]), layer
        assert np.array_equal(aux["k"].cpu().numpy().astype(np.int64), ref["k"]), layer
        assert aux["lambda"].item() == ref["lambda"], layer
        from test_gpu_parity import within_tol
        yg = O.bf16_bits_to_f64(y.cpu().numpy().view(np.uint16))
        ok, worst = within_tol(yg, ref["y"], bf16_out=True)
        assert ok, (layer, worst)


_STACK48 = {}


def _stack48():
    from dynamic_any_precision_b200.stack import DeviceStack
    if "s" not in _STACK48:
        _STACK48["s"] = DeviceStack(W.QWEN3_STACK)
    return _STACK48["s"]


@pytest.mark.parametrize("step", [0, 1, 2, 255])
def test_stack48_decode_teacher_forced_sampled(step):
    # the 48-layer stack at decode batch 32, the budget of step s being targets[s % 3]: all 48
    # layers run on the GPU; a strided subset of layers is checked against the oracle on the
    # GPU's own layer inputs (all 32 tokens' decisions, 4 tokens' outputs)
    from dynamic_any_precision_b200.stack import initial_stream
    shape = W.QWEN3_STACK
    stack = _stack48()
    T = shape.tokens
    target = shape.targets[step % len(shape.targets)]
    h = torch.from_numpy(initial_stream(shape, T, step=10 + step)).cuda()
    rec = _run_stack_recording(stack, h, torch.tensor([target], dtype=torch.float64, device="cuda"), T, stack.n_layers)
    layers = sorted({(step * 5 + 11 * i) % stack.n_layers for i in range(4)} | {stack.n_layers - 1})
    for layer in layers:
        _check_layer_teacher_forced(shape, layer, rec[layer], target, [0, 9, 22, 31])


def test_stack48_prefill_teacher_forced_sampled():
    # the stack's 2048-token prefill at the stored rate runs on the tensor-core path; three layers
    # are checked on their GPU inputs: routing and allocation of all 2048 tokens, a strided
    # 16-token subset of outputs
    from dynamic_any_precision_b200.stack import initial_stream
    shape = W.QWEN3_STACK
    stack = _stack48()
    T = W.STACK_PREFILL_TOKENS
    h = torch.from_numpy(initial_stream(shape, T, step=0)).cuda()
    rec = _run_stack_recording(stack, h, torch.tensor([float(shape.kmax)], dtype=torch.float64, device="cuda"), T,
                               stack.n_layers)
    for layer in (0, 23, 47):
        _check_layer_teacher_forced(shape, layer, rec[layer], float(shape.kmax), list(range(3, T, 128)))
