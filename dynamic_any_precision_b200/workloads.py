"""Seeded synthetic workloads for the routed bitplane MoE layer.

This module holds the named layer shapes and the seeded input generators that
both the CUDA path and the fp64 oracle consume. It performs none of the
method's arithmetic (no quantisation, routing, allocation or FFN math): it only
draws random numbers and rounds them to the storage dtypes (fp32, bf16).

Shapes follow the model families the pages evaluate on
(DPA-MoE: A Runtime Precision Control Framework for MoE Inference, Abstract:
Qwen3-30B-A3B and DeepSeekMoE-16B). No checkpoint is used: every weight is
N(0, 0.02) and every activation N(0, 1).

Random streams are keyed, so any expert can be generated on its own:
  router weights        default_rng([seed, 0])
  routed expert e       default_rng([seed, 1, e])   draws gate, up, down in order
  shared expert s       default_rng([seed, 2, s])   draws gate, up, down in order
  tokens (x)            default_rng([seed, 3, step])
Layer l of a stack uses seed = base_seed * 1000 + l.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import numpy as np

FMT_UNIFORM = 0
FMT_BCQ = 1


@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    n_shared: int
    fmt: int          # FMT_UNIFORM (asymmetric codes) or FMT_BCQ (+-1 planes)
    bits: int         # B: stored planes
    kmin: int
    kmax: int
    group: int
    norm_topk: int    # 1: softmax over the selected logits; 0: over all experts
    tokens: int
    targets: Tuple[float, ...]
    seed: int
    layers: int = 1


TINY = LayerShape("tiny_h256_e8_top2", 256, 512, 8, 2, 0, FMT_UNIFORM, 4, 2, 4, 64, 1,
                  4, (3.0,), 0)
QWEN3_B1 = LayerShape("qwen3_30b_a3b_moe_decode_b1", 2048, 768, 128, 8, 0, FMT_UNIFORM, 4, 2, 4,
                      128, 1, 1, (2.5,), 1)
QWEN3_B64 = LayerShape("qwen3_30b_a3b_moe_decode_b64", 2048, 768, 128, 8, 0, FMT_UNIFORM, 4, 2, 4,
                       128, 1, 64, (2.0, 2.5, 3.0, 3.5, 4.0), 2)
DEEPSEEK_B16 = LayerShape("deepseekmoe_16b_moe_decode_b16_bcq", 2048, 1408, 64, 6, 2, FMT_BCQ, 3, 1,
                          3, 128, 0, 16, (2.0,), 3)
QWEN3_STACK = LayerShape("qwen3_30b_a3b_moe_stack48", 2048, 768, 128, 8, 0, FMT_UNIFORM, 4, 2, 4,
                         128, 1, 32, (2.0, 3.0, 4.0), 4, layers=48)
STACK_PREFILL_TOKENS = 2048
STACK_DECODE_STEPS = 256
# one layer of the stack's prefill on its own (read at the stored rate: all pairs k = kmax)
QWEN3_PREFILL = LayerShape("qwen3_30b_a3b_moe_prefill_t2048", 2048, 768, 128, 8, 0, FMT_UNIFORM, 4, 2, 4,
                           128, 1, STACK_PREFILL_TOKENS, (4.0, 3.0), 5)

ALL_SHAPES = (TINY, QWEN3_B1, QWEN3_B64, DEEPSEEK_B16, QWEN3_STACK, QWEN3_PREFILL)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_f32(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)


def router_weights(shape: LayerShape, seed: Optional[int] = None) -> np.ndarray:
    """Router matrix Wr [E][H] as bf16 bits."""
    rng = np.random.default_rng([shape.seed if seed is None else seed, 0])
    return f32_to_bf16_bits(_normal_f32(rng, (shape.n_experts, shape.hidden), 0.02))


def expert_weights(shape: LayerShape, e: int, seed: Optional[int] = None,
                   shared: bool = False) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """fp32 (gate [I][H], up [I][H], down [H][I]) of routed expert e (or shared expert e)."""
    rng = np.random.default_rng([shape.seed if seed is None else seed, 2 if shared else 1, e])
    H, I = shape.hidden, shape.inter
    gate = _normal_f32(rng, (I, H), 0.02)
    up = _normal_f32(rng, (I, H), 0.02)
    down = _normal_f32(rng, (H, I), 0.02)
    return gate, up, down


def all_expert_weights(shape: LayerShape, seed: Optional[int] = None, threads: int = 0):
    """Stacked fp32 weights of every routed expert: gate [E][I][H], up [E][I][H], down [E][H][I].
    Experts are drawn from their own keyed streams, so drawing them in parallel threads gives
    the same values as drawing them one by one."""
    from concurrent.futures import ThreadPoolExecutor
    import os
    E, H, I = shape.n_experts, shape.hidden, shape.inter
    gate = np.empty((E, I, H), np.float32)
    up = np.empty((E, I, H), np.float32)
    down = np.empty((E, H, I), np.float32)

    def fill(e):
        gate[e], up[e], down[e] = expert_weights(shape, e, seed)

    n = threads or min(16, os.cpu_count() or 1)
    if n <= 1 or E <= 2:
        for e in range(E):
            fill(e)
    else:
        with ThreadPoolExecutor(n) as ex:
            list(ex.map(fill, range(E)))
    return gate, up, down


def shared_weights_bf16(shape: LayerShape, seed: Optional[int] = None):
    """Shared (always-on) experts as dense bf16 bits: gate [S][I][H], up [S][I][H], down [S][H][I]."""
    S, H, I = shape.n_shared, shape.hidden, shape.inter
    g = np.empty((S, I, H), np.uint16)
    u = np.empty((S, I, H), np.uint16)
    d = np.empty((S, H, I), np.uint16)
    for s in range(S):
        a, b, c = expert_weights(shape, s, seed, shared=True)
        g[s], u[s], d[s] = f32_to_bf16_bits(a), f32_to_bf16_bits(b), f32_to_bf16_bits(c)
    return g, u, d


def tokens(shape: LayerShape, n_tokens: Optional[int] = None, step: int = 0,
           seed: Optional[int] = None) -> np.ndarray:
    """Activations x [T][H] as bf16 bits, N(0, 1)."""
    T = shape.tokens if n_tokens is None else n_tokens
    rng = np.random.default_rng([shape.seed if seed is None else seed, 3, step])
    return f32_to_bf16_bits(rng.standard_normal((T, shape.hidden), dtype=np.float32))


def layer_seed(shape: LayerShape, layer: int) -> int:
    return shape.seed * 1000 + layer


def shape_by_name(name: str) -> LayerShape:
    for s in ALL_SHAPES:
        if s.name == name:
            return s
    raise KeyError(name)


def with_sizes(shape: LayerShape, **kw) -> LayerShape:
    return dataclasses.replace(shape, **kw)


__all__: List[str] = [n for n in dir() if not n.startswith("_")]
