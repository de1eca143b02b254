"""Oracle work for the parity tests, runnable in a spawned process pool. Every input is drawn
from the seeded generators; nothing here reads a result of the CUDA path."""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

from dynamic_any_precision_b200 import workloads as W
from oracle import dpa_oracle as O

_POOL = None


def pool() -> ProcessPoolExecutor:
    global _POOL
    if _POOL is None:
        n = max(1, min(16, (os.cpu_count() or 2) - 1))
        _POOL = ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"))
    return _POOL


def encode_expert_job(shape, e, seed=None):
    g, u, d = W.expert_weights(shape, e, seed)
    return e, O.encode_expert(g, u, d, shape.fmt, shape.bits, shape.group)


def encode_experts(shape, experts, seed=None):
    experts = sorted(set(int(e) for e in experts))
    if len(experts) <= 2:
        return dict(encode_expert_job(shape, e, seed) for e in experts)
    futs = [pool().submit(encode_expert_job, shape, e, seed) for e in experts]
    return dict(f.result() for f in futs)


def reference_layer(shape, x_bits, target, token_subset=None, seed=None):
    """Oracle forward of one layer: route, encode the routed experts, allocate, FFN, combine."""
    wr = W.router_weights(shape, seed)
    idx, gates, logits = O.route(x_bits, wr, shape.top_k, shape.norm_topk)
    experts = encode_experts(shape, np.unique(idx), seed)
    r = np.full((shape.n_experts, shape.bits), np.nan)
    for e, enc in experts.items():
        r[e] = enc["r"]
    shared = W.shared_weights_bf16(shape, seed) if shape.n_shared else None
    y, aux = O.moe_forward(x_bits, wr, experts, shape, target, shared=shared, r_table=r, logits=logits,
                           token_subset=token_subset)
    aux["experts"] = experts
    aux["r"] = r
    return y, aux


def pair_outputs(shape, x_bits, aux, pairs):
    """Oracle expert output o (before gate weighting) for the listed (t, slot) pairs."""
    x = O.bf16_bits_to_f64(x_bits)
    out = {}
    for t, j in pairs:
        e, k = int(aux["idx"][t, j]), int(aux["k"][t, j])
        wg, wu, wd = O.dequant_expert(aux["experts"][e], shape.fmt, shape.bits, k, shape.group)
        out[(t, j)] = O.expert_ffn(x[t], wg, wu, wd)
    return out
