"""dpa_route_noalloc: the router entry point that allocates nothing, for callers that cannot
call cudaMalloc (an engine that owns all device memory, a loop that must stay clear of the
allocator). It must make exactly the decisions dpa_route makes. Collected last on purpose."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from dynamic_any_precision_b200 import dpa, workloads as W  # noqa: E402

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    fn = dpa.lib().dpa_route_noalloc
    fn.argtypes = [ctypes.POINTER(dpa.LayerDesc), ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


@pytest.mark.parametrize("shape,T", [(W.QWEN3_B1, 7), (W.DEEPSEEK_B16, 16), (W.TINY, 4)])
def test_route_noalloc_matches_route_on_two_calls_in_a_row(shape, T):
    fn = _noalloc_fn()
    desc = dpa.make_desc(shape)
    wr = torch.from_numpy(W.router_weights(shape).view(np.int16)).cuda()
    ws = dpa.new_workspace(desc, T)
    for step in (21, 22):   # two calls in a row, different tokens: the shared scratch is reused
        x = torch.from_numpy(W.tokens(shape, T, step=step).view(np.int16)).cuda()
        ref_logits = torch.empty((T, shape.n_experts), dtype=torch.float64, device="cuda")
        ref_idx, ref_gate = dpa.route(desc, x, wr, ws, logits=ref_logits)
        idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
        gate = torch.empty((T, shape.top_k), dtype=torch.float64, device="cuda")
        logits = torch.empty((T, shape.n_experts), dtype=torch.float64, device="cuda")
        st = fn(ctypes.byref(desc), x.data_ptr(), T, wr.data_ptr(), idx.data_ptr(), gate.data_ptr(),
                logits.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0
        torch.cuda.synchronize()
        assert dpa.device_status(ws) == 0
        # routing is bit-exact in every test of this suite, so the comparison is equality
        assert torch.equal(idx, ref_idx)
        assert torch.equal(gate, ref_gate)
        assert torch.equal(logits, ref_logits)


@pytest.mark.parametrize("T", [128, 512])
def test_route_noalloc_large_batches_against_oracle(T):
    # from 128 tokens on dpa_route switches to its tiled kernels while this entry point keeps the
    # per-logit kernel; 512 tokens x 128 experts fills its logits scratch exactly. Decisions must
    # equal the oracle's bit for bit, and dpa_route's, on two calls in a row.
    from oracle_jobs import route_parallel
    shape = W.QWEN3_B64
    fn = _noalloc_fn()
    desc = dpa.make_desc(shape)
    wr = torch.from_numpy(W.router_weights(shape).view(np.int16)).cuda()
    ws = dpa.new_workspace(desc, T)
    for step in (31, 32):
        xb = W.tokens(shape, T, step=step)
        x = torch.from_numpy(xb.view(np.int16)).cuda()
        idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
        gate = torch.empty((T, shape.top_k), dtype=torch.float64, device="cuda")
        logits = torch.empty((T, shape.n_experts), dtype=torch.float64, device="cuda")
        st = fn(ctypes.byref(desc), x.data_ptr(), T, wr.data_ptr(), idx.data_ptr(), gate.data_ptr(),
                logits.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0
        torch.cuda.synchronize()
        ridx, rg, rl = route_parallel(shape, xb)
        assert np.array_equal(logits.cpu().numpy(), rl)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        assert np.array_equal(gate.cpu().numpy(), rg)
        ref_idx, ref_gate = dpa.route(desc, x, wr, ws)
        assert dpa.device_status(ws) == 0
        assert torch.equal(idx, ref_idx) and torch.equal(gate, ref_gate)


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    fn = _noalloc_fn()
    desc = dpa.make_desc(W.QWEN3_B1)
    buf = torch.zeros(16, dtype=torch.float64, device="cuda")
    p = buf.data_ptr()
    # 600 tokens x 128 experts exceeds the fixed logits scratch; 2000 tokens exceeds the counters
    assert fn(ctypes.byref(desc), p, 600, p, p, p, None, None) == 2
    assert fn(ctypes.byref(desc), p, 2000, p, p, p, None, None) == 2
