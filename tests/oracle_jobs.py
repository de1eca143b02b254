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


# Encoded experts already computed in this process, keyed by everything that determines them
# (the expert's random stream and the encoding parameters), so that tests sharing a layer encode
# each of its experts once.
_ENC_CACHE = {}
_ENC_CACHE_MAX = 300


def _enc_key(shape, e, seed):
    return (shape.seed if seed is None else seed, int(e), shape.hidden, shape.inter, shape.fmt, shape.bits,
            shape.group)


def encode_experts(shape, experts, seed=None):
    experts = sorted(set(int(e) for e in experts))
    out = {e: _ENC_CACHE[_enc_key(shape, e, seed)] for e in experts if _enc_key(shape, e, seed) in _ENC_CACHE}
    todo = [e for e in experts if e not in out]
    if len(todo) <= 2:
        new = dict(encode_expert_job(shape, e, seed) for e in todo)
    else:
        futs = [pool().submit(encode_expert_job, shape, e, seed) for e in todo]
        new = dict(f.result() for f in futs)
    if len(_ENC_CACHE) + len(new) > _ENC_CACHE_MAX:
        _ENC_CACHE.clear()
    for e, enc in new.items():
        _ENC_CACHE[_enc_key(shape, e, seed)] = enc
    out.update(new)
    return out


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


# ----------------------------------------------------------------------------- full-size helpers
# The same oracle functions, spread over the spawned pool: routing by token chunks (each token is
# routed on its own), residual tables and expert outputs by expert (a worker encodes the expert
# from its seeded stream and keeps it for later jobs of the same process).

_WORKER_ENC = {}


def _worker_encoded(shape, e, seed):
    key = _enc_key(shape, e, seed)
    if key not in _WORKER_ENC:
        if len(_WORKER_ENC) >= 48:
            _WORKER_ENC.clear()
        _WORKER_ENC[key] = encode_expert_job(shape, e, seed)[1]
    return _WORKER_ENC[key]


def _route_chunk_job(x_bits, wr, K, norm_topk):
    return O.route(x_bits, wr, K, norm_topk)


def _rtable_job(shape, e, seed):
    return e, _worker_encoded(shape, e, seed)["r"]


def _pair_outputs_job(shape, e, seed, rows):
    """rows: list of (key, k, x_row fp64) -> {key: expert output at k planes}."""
    enc = _worker_encoded(shape, e, seed)
    dense = {}
    out = {}
    for key, k, xr in rows:
        if k not in dense:
            dense[k] = O.dequant_expert(enc, shape.fmt, shape.bits, k, shape.group)
        out[key] = O.expert_ffn(xr, *dense[k])
    return out


def route_parallel(shape, x_bits, seed=None, chunk=16):
    wr = W.router_weights(shape, seed)
    T = x_bits.shape[0]
    if T <= chunk:
        return O.route(x_bits, wr, shape.top_k, shape.norm_topk)
    futs = [pool().submit(_route_chunk_job, x_bits[a:a + chunk], wr, shape.top_k, shape.norm_topk)
            for a in range(0, T, chunk)]
    parts = [f.result() for f in futs]
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]),
            np.concatenate([p[2] for p in parts]))


def residual_tables(shape, experts, seed=None):
    """r [E][B] with the rows of the listed experts filled (others NaN)."""
    r = np.full((shape.n_experts, shape.bits), np.nan)
    experts = sorted(set(int(e) for e in experts))
    cached = [e for e in experts if _enc_key(shape, e, seed) in _ENC_CACHE]
    for e in cached:
        r[e] = _ENC_CACHE[_enc_key(shape, e, seed)]["r"]
    futs = [pool().submit(_rtable_job, shape, e, seed) for e in experts if e not in cached]
    for f in futs:
        e, re_ = f.result()
        r[e] = re_
    return r


def reference_layer_parallel(shape, x_bits, target, token_subset, seed=None, logits=None):
    """Oracle forward of one layer at full size: routing and allocation of every token, the
    expert FFNs and combine of the tokens in token_subset (other rows NaN)."""
    if logits is None:
        idx, gates, logits = route_parallel(shape, x_bits, seed)
    else:
        idx, gates, logits = O.route(x_bits, None, shape.top_k, shape.norm_topk, logits=logits)
    r = residual_tables(shape, np.unique(idx), seed)
    k, lam = O.allocate(idx, gates, r, shape.kmin, shape.kmax, target)
    x = O.bf16_bits_to_f64(x_bits)
    by_expert = {}
    for t in token_subset:
        for j in range(shape.top_k):
            by_expert.setdefault(int(idx[t, j]), []).append(((t, j), int(k[t, j]), x[t]))
    futs = [pool().submit(_pair_outputs_job, shape, e, seed, rows) for e, rows in by_expert.items()]
    outs = {}
    for f in futs:
        outs.update(f.result())
    shared = W.shared_weights_bf16(shape, seed) if shape.n_shared else None
    y = np.full((x_bits.shape[0], shape.hidden), np.nan)
    for t in token_subset:
        y[t] = O.combine_token(gates[t], [outs[(t, j)] for j in range(shape.top_k)],
                               O.shared_outputs(x[t], shared))
    return y, {"idx": idx, "gates": gates, "logits": logits, "k": k, "lambda": lam, "r": r, "pair_out": outs}
