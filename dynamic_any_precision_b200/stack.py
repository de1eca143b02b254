"""A stack of routed bitplane MoE layers resident on one GPU.

Per layer l: x = bf16(RMSNorm(h)); y = MoE_l(x); h += y, with the fp32 residual stream h.
Every step runs in the CUDA library (dpa_residual_rmsnorm, dpa_moe_forward); this module only
builds the layers (seeded synthetic weights, host encoder) and sequences the calls.
"""
from __future__ import annotations

from typing import List, Optional

import numpy as np

from . import dpa
from . import workloads as W


class DeviceStack:
    def __init__(self, shape: W.LayerShape, n_layers: Optional[int] = None, device="cuda", threads: int = 0):
        self.shape = shape
        self.desc = dpa.make_desc(shape)
        self.n_layers = shape.layers if n_layers is None else n_layers
        self.layers: List[dpa.DeviceLayer] = []
        for layer in range(self.n_layers):
            seed = W.layer_seed(shape, layer)
            g, u, d = W.all_expert_weights(shape, seed, threads=threads)
            planes, meta, r = dpa.encode(self.desc, g, u, d, n_threads=threads)
            del g, u, d
            wr = W.router_weights(shape, seed)
            sh = W.shared_weights_bf16(shape, seed) if shape.n_shared else None
            self.layers.append(dpa.DeviceLayer.from_host(self.desc, planes, meta, r, wr, sh, device=device))

    def buffers(self, n_tokens: int, device="cuda"):
        """Workspace and activation buffers for `n_tokens` tokens."""
        import torch
        H = self.shape.hidden
        return {"ws": dpa.new_workspace(self.desc, n_tokens, device=device),
                "x": torch.empty((n_tokens, H), dtype=torch.int16, device=device),
                "y": torch.empty((n_tokens, H), dtype=torch.int16, device=device)}

    def forward(self, h, target, bufs, aux_per_layer=None, stream=None):
        """Run every layer on the residual stream h (fp32 [T][H], updated in place).
        target: CUDA fp64 scalar tensor. aux_per_layer: optional list of aux dicts.
        Returns x, the normalised input the next layer would read."""
        x, y, ws = bufs["x"], bufs["y"], bufs["ws"]
        dpa.residual_rmsnorm(h, x, None, stream=stream)
        for i, layer in enumerate(self.layers):
            aux = aux_per_layer[i] if aux_per_layer is not None else None
            dpa.moe_forward(layer, x, target, ws, y=y, aux=aux, stream=stream)
            dpa.residual_rmsnorm(h, x, y, stream=stream)
        return x


def initial_stream(shape: W.LayerShape, n_tokens: int, step: int = 0) -> np.ndarray:
    """Seeded fp32 residual stream to start from: the bf16 token activations, widened."""
    return W.bf16_bits_to_f32(W.tokens(shape, n_tokens, step=step)).astype(np.float32)
