"""Device-side failure handling, in the forms that fault, trap or hang nothing: bounded waits that
run out against a barrier nothing completes (short limits), and invalid device data (NaN/Inf
tokens, out-of-range expert ids). Each is reported through the workspace's error flag and read
with dpa_device_status; the context stays usable afterwards."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from dynamic_any_precision_b200 import dpa, workloads as W  # noqa: E402
from test_gpu_parity import GpuLayer  # noqa: E402

pytestmark = pytest.mark.gpu

TIMEOUT, INVALID = 5, 6


def _tiny_forward_ok(gl, x_bits):
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    tg = torch.tensor([3.0], dtype=torch.float64, device="cuda")
    ws = dpa.new_workspace(gl.desc, x.shape[0])
    y1 = dpa.moe_forward(gl.layer, x, tg, ws).clone()
    y2 = dpa.moe_forward(gl.layer, x, tg, ws)
    assert dpa.device_status(ws) == 0
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("kind", [0, 1, 2])
def test_bounded_wait_runs_out_and_is_reported(kind):
    gl = GpuLayer.get(W.TINY)
    x = W.tokens(W.TINY, 4, step=2)
    ws = dpa.new_workspace(gl.desc, 4)
    st = dpa.lib().dpa_debug_timeout_probe(ws.data_ptr(), ws.numel(), kind, 2_000_000,
                                           torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert dpa.device_status(ws) == TIMEOUT
    assert dpa.device_status(ws) == 0            # read and cleared
    _tiny_forward_ok(gl, x)                      # the context is still usable


def test_timeout_probe_rejects_bad_arguments():
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    L = dpa.lib()
    assert L.dpa_debug_timeout_probe(ws.data_ptr(), ws.numel(), 3, 2_000_000, s) == 1
    assert L.dpa_debug_timeout_probe(ws.data_ptr(), ws.numel(), 0, 10, s) == 1
    assert L.dpa_debug_timeout_probe(ws.data_ptr(), 100, 0, 2_000_000, s) == 1


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")])
@pytest.mark.parametrize("T", [3, 130])
def test_non_finite_tokens_set_the_device_flag(bad, T):
    # per-logit router (3 tokens) and tiled router (130 tokens)
    shape = W.TINY
    d = dpa.make_desc(shape)
    x = W.tokens(shape, T, step=5).copy()
    x[T // 2, 17] = W.f32_to_bf16_bits(np.array([bad], dtype=np.float32))[0]
    wr = torch.from_numpy(W.router_weights(shape).view(np.int16)).cuda()
    ws = dpa.new_workspace(d, T)
    dpa.route(d, torch.from_numpy(x.view(np.int16)).cuda(), wr, ws)
    assert dpa.device_status(ws) == INVALID
    _tiny_forward_ok(GpuLayer.get(shape), W.tokens(shape, 4, step=6))


@pytest.mark.parametrize("bad_e", [8, -1, 1 << 20])
def test_out_of_range_expert_id_in_allocate(bad_e):
    shape = W.TINY
    d = dpa.make_desc(shape)
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(8, 2, replace=False) for _ in range(4)]).astype(np.int32)
    idx[2, 1] = bad_e
    g = -np.sort(-rng.dirichlet(np.ones(2), size=4), axis=1)
    r = np.ones((8, 4))
    ws = dpa.new_workspace(d, 4)
    k0 = torch.full((4, 2), 7, dtype=torch.uint8, device="cuda")
    st = dpa.lib().dpa_allocate(dpa.ctypes.byref(d), torch.from_numpy(r).cuda().data_ptr(),
                                torch.from_numpy(idx).cuda().data_ptr(), torch.from_numpy(g).cuda().data_ptr(), 4,
                                torch.tensor([3.0], dtype=torch.float64, device="cuda").data_ptr(), k0.data_ptr(),
                                None, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert dpa.device_status(ws) == INVALID
    assert torch.all(k0 == 7)
