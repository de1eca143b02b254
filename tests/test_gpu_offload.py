"""Host-to-device prefix streaming of offloaded experts (nested bitplanes read by prefix): a
device layer whose bytes are all poisoned, then filled only with the streamed first kmax_e planes
(and their scale data) of the experts a step routes to, gives exactly the outputs of the fully
resident layer."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from dynamic_any_precision_b200 import dpa, workloads as W  # noqa: E402
from test_gpu_parity import GpuLayer  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,T,target", [(W.QWEN3_B1, 1, 2.5), (W.QWEN3_B64, 16, 3.0),
                                            (W.DEEPSEEK_B16, 16, 2.0)])
def test_streamed_prefixes_reproduce_the_resident_layer(shape, T, target):
    gl = GpuLayer.get(shape)
    d = gl.desc
    host_planes = torch.from_numpy(gl.planes_host).pin_memory()
    host_meta = gl.layer.meta.cpu().pin_memory()
    x = torch.from_numpy(W.tokens(shape, T, step=91).view(np.int16)).cuda()
    tg = torch.tensor([target], dtype=torch.float64, device="cuda")
    ws = dpa.new_workspace(d, T)
    y_res = dpa.moe_forward(gl.layer, x, tg, ws).clone()
    # decisions of the step (route + allocate on the device), read back
    idx, gate = dpa.route(d, x, gl.layer.w_router, ws)
    k, _ = dpa.allocate(d, gl.layer.rtable, idx, gate, tg, ws)
    idx_h, k_h = idx.cpu().numpy(), k.cpu().numpy()
    kmax = {}
    for e, kk in zip(idx_h.reshape(-1).tolist(), k_h.reshape(-1).tolist()):
        kmax[e] = max(kmax.get(e, 0), kk)
    # a device layer holding nothing but poison
    dev = dpa.DeviceLayer(d, torch.full_like(gl.layer.planes, 0xA5), torch.full_like(gl.layer.meta, 0xFF),
                          gl.layer.rtable, gl.layer.w_router, gl.layer.shared)
    experts = sorted(kmax)
    nbytes = dpa.stream_prefixes(d, host_planes, host_meta, experts, [kmax[e] for e in experts], dev.planes, dev.meta)
    s = dpa.encoded_sizes(d)
    plane = shape.hidden * shape.inter // 8
    want = sum(3 * kmax[e] * plane for e in experts)
    if shape.fmt == W.FMT_UNIFORM:
        want += len(experts) * s.meta_per_expert
    else:
        want += sum(kmax[e] * 3 * shape.inter * (shape.hidden // shape.group) * 2 for e in experts)
    assert nbytes == want
    assert nbytes < len(experts) * (s.planes_per_expert + s.meta_per_expert) or target == shape.kmax
    y_str = dpa.moe_forward(dev, x, tg, ws)
    assert dpa.device_status(ws) == 0
    assert torch.equal(y_str, y_res)


def test_stream_prefixes_rejects_bad_arguments():
    gl = GpuLayer.get(W.TINY)
    d = gl.desc
    hp = torch.from_numpy(gl.planes_host)
    hm = gl.layer.meta.cpu()
    for ex, kp in (([8], [2]), ([-1], [2]), ([0], [0]), ([0], [5])):
        with pytest.raises(dpa.DpaError, match="INVALID_ARG"):
            dpa.stream_prefixes(d, hp, hm, ex, kp, gl.layer.planes, gl.layer.meta)
