#!/usr/bin/env python
"""Benchmark: MoE-layer decode tokens/s at a target bits-per-weight, and the HBM bandwidth of
the planes the variable-plane expert GEMV reads, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dpa|reference] [--workload NAME]

A step is one pass of the whole hot path over one batch of synthetic tokens: route (exact-dot
softmax top-k), plane allocation (64-step Lagrangian bisection), grouping by (expert, k), the
gate/up GEMV with SwiGLU, the down GEMV and the gate-weighted combine - one dpa_moe_forward.
Inputs are resident in HBM when the timed region starts. The layer is encoded once and copied
`--copies` times in device memory; step i uses copy i % copies and its own tokens, so no weight
byte is re-read within copies-1 steps and the L2 cache (126 MB) cannot serve the planes.
The K timed steps are one CUDA graph without instrumentation; a second graph of the same K
steps with CUDA events at the stage boundaries gives the per-kernel device times.

N > 1 GPUs run independent replicas (no collective on the data path; the path shards by
token batch), one process per GPU under torchrun; the time is the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores (rank 0 only), each step a
bounded sample of the same workload (see cpu_baseline in the output).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_any_precision_b200 import workloads as W  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1400.0   # sustained bf16 under the power cap, an earlier measurement on this machine


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1024)
    ap.add_argument("--warmup", type=int, default=32)
    ap.add_argument("--impl", choices=("dpa", "reference"), default="dpa")
    ap.add_argument("--workload", default=W.QWEN3_B64.name)
    ap.add_argument("--target", type=float, default=None)
    ap.add_argument("--no-sweep", action="store_true",
                    help="time only the headline budget (the batch-64 workload sweeps all its budgets)")
    ap.add_argument("--copies", type=int, default=16)
    ap.add_argument("--e2e-steps", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--offload", action="store_true",
                    help="experts resident in pinned host memory: every step streams the planes it reads "
                         "(first kmax_e planes per routed expert) host->device before the layer runs, and "
                         "the same steps are timed again streaming every stored plane")
    ap.add_argument("--cpu-sample-pairs", type=int, default=24,
                    help="expert FFN pairs the CPU-baseline sample times (round robin over the steps)")
    return ap.parse_args(argv)


# The headline budget of each workload: the batch-64 layer is quoted at 3.0 bpw, the middle of
# its sweep; the others at their first (or only) budget.
HEADLINE_TARGET = {W.QWEN3_B64.name: 3.0}


def headline_target(shape):
    return HEADLINE_TARGET.get(shape.name, shape.targets[0])


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _peaks():
    """All measured peaks as a dict (empty when the file is absent)."""
    try:
        with open(PEAKS_PATH) as f:
            return json.load(f)
    except Exception:
        return {}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) in a thread."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples = []
        self.ok = False
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                try:
                    rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# ----------------------------------------------------------------------------- workload

def build_layer(shape, seed=None):
    """Encode one layer on the host (product encoder)."""
    from dynamic_any_precision_b200 import dpa
    desc = dpa.make_desc(shape)
    g, u, d = W.all_expert_weights(shape, seed)
    planes, meta, r = dpa.encode(desc, g, u, d)
    del g, u, d
    wr = W.router_weights(shape, seed)
    sh = W.shared_weights_bf16(shape, seed) if shape.n_shared else None
    return desc, planes, meta, r, wr, sh


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the dominant
# kernel, from one ncu capture of the current kernel code (the capture commands and figures are
# kept with the profile summaries). Workloads without such a capture report null.
NCU_TRAFFIC_BYTES = {
    ("qwen3_30b_a3b_moe_decode_b64", 3.0): 172_652_288,         # vp_gemv_kernel<0,4,2,2> (gate/up)
    ("qwen3_30b_a3b_moe_prefill_t2048", 4.0): 301_577_728,      # gemm_tc_kernel<0,4> (gate/up)
}


def max_over_ranks(dist, values, device):
    """Element-wise maximum of per-rank device times (ms) over all ranks (every rank gets it);
    the values unchanged when there is one process."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    tt = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return [float(v) for v in tt.tolist()]


def replica_token_seed(rank: int, step: int) -> int:
    """Seed of the synthetic tokens of one step on one rank: distinct per rank and step."""
    return 1_000_000 * rank + step


def algorithmic_bytes(shape, idx, k):
    """Bytes the gate/up and down GEMVs must read for one step: for every active expert its first
    kmax_e planes of each matrix plus its scale data (kmax_e = max k over its pairs)."""
    H, I, G, B = shape.hidden, shape.inter, shape.group, shape.bits
    plane = H * I // 8
    kmax = {}
    for e, kk in zip(idx.reshape(-1).tolist(), k.reshape(-1).tolist()):
        kmax[e] = max(kmax.get(e, 0), kk)
    gu = dn = 0
    for e, km in kmax.items():
        if shape.fmt == W.FMT_UNIFORM:
            gu += 2 * km * plane + 2 * I * (H // G) * 4
            dn += km * plane + H * (I // G) * 4
        else:
            gu += 2 * km * plane + 2 * km * I * (H // G) * 2
            dn += km * plane + km * H * (I // G) * 2
    return gu, dn, len(kmax)


def run_dpa(args, shape, targets, rank, world, dist):
    """Times K graph-replayed steps at each budget in `targets` (the budget is a device scalar, so
    one captured graph serves them all). Returns one result dict per budget."""
    import torch
    from dynamic_any_precision_b200 import dpa

    dev = torch.device("cuda", torch.cuda.current_device())
    desc, planes, meta, r, wr, sh = build_layer(shape)
    T, K = shape.tokens, shape.top_k
    L = max(1, args.copies)
    base = dpa.DeviceLayer.from_host(desc, planes, meta, r, wr, sh, device=dev)
    layers = [base]
    for _ in range(L - 1):
        layers.append(dpa.DeviceLayer(desc, base.planes.clone(), base.meta.clone(), base.rtable.clone(),
                                      base.w_router.clone(), base.shared))
    n_total = args.warmup + args.steps
    # distinct tokens per step (and per rank)
    xs = np.stack([W.tokens(shape, T, step=replica_token_seed(rank, i)) for i in range(n_total)])
    x_dev = torch.from_numpy(xs.view(np.int16)).to(dev)
    y_dev = torch.empty((n_total, T, shape.hidden), dtype=torch.int16, device=dev)
    tg = torch.tensor([targets[0]], dtype=torch.float64, device=dev)
    ws = dpa.new_workspace(desc, T, device=dev)
    idx_all = torch.empty((args.steps, T, K), dtype=torch.int32, device=dev)
    gate_all = torch.empty((args.steps, T, K), dtype=torch.float64, device=dev)
    k_all = torch.empty((args.steps, T, K), dtype=torch.uint8, device=dev)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    for row in events:          # torch creates events lazily: record once so the handles exist
        for ev in row:
            ev.record()

    def step(i, timed_j=None):
        aux = None
        if timed_j is not None:
            aux = {"topk_idx": idx_all[timed_j], "topk_gate": gate_all[timed_j], "k": k_all[timed_j],
                   "events": events[timed_j]}
        dpa.moe_forward(layers[i % L], x_dev[i], tg, ws, y=y_dev[i], aux=aux)

    # eager run of every distinct layer copy once (loads the module, sets kernel attributes)
    for i in range(min(L, n_total)):
        step(i)
    torch.cuda.synchronize()
    assert dpa.device_status(ws) == 0

    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    g_warm, g_timed, g_stages = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g_warm, stream=s):
            for i in range(args.warmup):
                step(i)
        # the timed region: K steps, no instrumentation inside
        with torch.cuda.graph(g_timed, stream=s):
            for j in range(args.steps):
                step(args.warmup + j)
        # the same K steps again with stage events, for per-kernel device times
        with torch.cuda.graph(g_stages, stream=s):
            for j in range(args.steps):
                step(args.warmup + j, timed_j=j)
    torch.cuda.synchronize()

    names = ["route", "allocate", "shared", "gateup", "down", "combine"]
    results = []
    for target in targets:
        tg.fill_(target)
        # untimed: the warm-up steps, then one whole replay of the timed graph itself (its upload
        # and first launch stay outside the measurement)
        g_warm.replay()
        g_timed.replay()
        torch.cuda.synchronize()
        assert dpa.device_status(ws) == 0

        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(torch.cuda.current_device()) as clk:
            t0.record()
            g_timed.replay()
            t1.record()
            torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        ms = t0.elapsed_time(t1)
        st = dpa.device_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {dpa.STATUS_NAMES.get(st, st)}")
        ms = max_over_ranks(dist, [ms], dev)[0]

        # per-stage kernel times: the same steps replayed once more with stage events
        g_stages.replay()
        torch.cuda.synchronize()
        assert dpa.device_status(ws) == 0
        stage_ms = {n: 0.0 for n in names}
        for j in range(args.steps):
            ev = events[j]
            for q, n in enumerate(names):
                stage_ms[n] += ev[q].elapsed_time(ev[q + 1])
        idx_h, k_h = idx_all.cpu().numpy(), k_all.cpu().numpy()
        gu_bytes = dn_bytes = 0
        n_active = 0
        for j in range(args.steps):
            a, b, c = algorithmic_bytes(shape, idx_h[j], k_h[j])
            gu_bytes += a
            dn_bytes += b
            n_active += c
        mean_bpw = float(k_h.astype(np.float64).mean())
        results.append({"target": target, "ms": ms, "stage_ms": stage_ms, "gu_bytes": gu_bytes, "dn_bytes": dn_bytes,
                        "n_active": n_active, "mean_bpw": mean_bpw, "clocks": clk.summary()})

    # e2e through the public API with host buffers (pinned), copies inside the timed region, at the
    # first (headline) budget
    tg.fill_(targets[0])
    e2e = None
    if args.e2e_steps > 0:
        n_e = min(args.e2e_steps, n_total)
        x_host = torch.from_numpy(xs[:n_e].view(np.int16)).pin_memory()
        y_host = torch.empty((n_e, T, shape.hidden), dtype=torch.int16).pin_memory()
        x_buf = torch.empty((T, shape.hidden), dtype=torch.int16, device=dev)
        y_buf = torch.empty((T, shape.hidden), dtype=torch.int16, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for i in range(n_e):
            x_buf.copy_(x_host[i], non_blocking=True)
            dpa.moe_forward(layers[i % L], x_buf, tg, ws, y=y_buf)
            y_host[i].copy_(y_buf, non_blocking=True)
            torch.cuda.current_stream().synchronize()   # the host reads this step's result
        e1.record()
        torch.cuda.synchronize()
        e_ms = e0.elapsed_time(e1)
        e_ms = max_over_ranks(dist, [e_ms], dev)[0]
        e2e = {"value": world * T * n_e / (e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(x_buf.numel() * 2), "d2h_bytes_per_step": int(y_buf.numel() * 2),
               "steps": n_e}

    P = T * K
    tc = (shape.fmt == dpa.FMT_UNIFORM and shape.hidden % 256 == 0 and shape.inter % 256 == 0 and
          P >= 16 * shape.n_experts)
    # route (1, or 3 from 128 tokens), allocate (1, or 2 above 2048 pairs), the expert FFN (3: gate/up,
    # h digits, down; or 3 on the tensor-core path: row permute, two GEMMs), combine, shared experts (2)
    launches_per_step = ((3 if T >= 128 else 1) + (2 if P > 2048 else 1) + 3 + 1 + (2 if shape.n_shared else 0))
    for res in results:
        res.update({"tc": tc, "e2e": e2e, "launches": launches_per_step * args.steps})
    return results


def run_offload(args, shape, target, rank, world, dist):
    """Experts offloaded to pinned host memory. A step routes and allocates on the device, reads
    the decisions back (the host must know what to fetch), streams the first kmax_e planes of
    every routed expert host->device (one copy per matrix prefix), and runs the layer on the
    device copy, which holds nothing else. The same steps are then timed streaming all stored
    planes. Time per step is device time between events (host synchronisations inside)."""
    import torch
    from dynamic_any_precision_b200 import dpa

    dev = torch.device("cuda", torch.cuda.current_device())
    desc, planes, meta, r, wr, sh = build_layer(shape)
    T, K = shape.tokens, shape.top_k
    host_planes = torch.from_numpy(planes).pin_memory()
    host_meta = torch.from_numpy(meta).pin_memory()
    layer = dpa.DeviceLayer.from_host(desc, planes, meta, r, wr, sh, device=dev)
    n_total = args.warmup + args.steps
    xs = [torch.from_numpy(W.tokens(shape, T, step=replica_token_seed(rank, i)).view(np.int16)).to(dev)
          for i in range(n_total)]
    tg = torch.tensor([target], dtype=torch.float64, device=dev)
    ws = dpa.new_workspace(desc, T, device=dev)
    y = torch.empty((T, shape.hidden), dtype=torch.int16, device=dev)
    out = {}
    for mode in ("prefix", "full"):
        total_ms, total_bytes = 0.0, 0
        for i in range(n_total):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            idx, gate = dpa.route(desc, xs[i], layer.w_router, ws)
            k, _ = dpa.allocate(desc, layer.rtable, idx, gate, tg, ws)
            idx_h, k_h = idx.cpu().numpy().reshape(-1), k.cpu().numpy().reshape(-1)
            kmax = {}
            for e, kk in zip(idx_h.tolist(), k_h.tolist()):
                kmax[e] = max(kmax.get(e, 0), kk)
            ex = sorted(kmax)
            kp = [kmax[e] if mode == "prefix" else shape.bits for e in ex]
            nb = dpa.stream_prefixes(desc, host_planes, host_meta, ex, kp, layer.planes, layer.meta)
            dpa.moe_forward(layer, xs[i], tg, ws, y=y)
            e1.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                total_ms += e0.elapsed_time(e1)
                total_bytes += nb
        assert dpa.device_status(ws) == 0
        ms = max_over_ranks(dist, [total_ms], dev)[0]
        out[mode] = {"ms_per_step": ms / args.steps, "tokens_per_s": world * T * args.steps / (ms * 1e-3),
                     "h2d_bytes_per_step": total_bytes / args.steps,
                     "h2d_gbs": total_bytes / (ms * 1e-3) / 1e9}
    return out


def run_stack(args, shape, rank, world, dist):
    """48-layer stack: one prefill pass at the stored rate, then decode steps of fresh tokens
    with the budget cycling over the shape's targets (one captured graph per budget)."""
    import torch
    from dynamic_any_precision_b200 import dpa
    from dynamic_any_precision_b200.stack import DeviceStack, initial_stream

    dev = torch.device("cuda", torch.cuda.current_device())
    t_build = time.time()
    stack = DeviceStack(shape, device=dev)
    build_s = time.time() - t_build
    T, H = shape.tokens, shape.hidden
    Tp = W.STACK_PREFILL_TOKENS
    bufs = stack.buffers(max(T, Tp), device=dev)
    small = {"ws": bufs["ws"], "x": bufs["x"][:T], "y": bufs["y"][:T]}
    tgs = [torch.tensor([t], dtype=torch.float64, device=dev) for t in shape.targets]
    n_total = args.warmup + args.steps
    h0 = torch.from_numpy(np.stack([initial_stream(shape, T, step=1_000_000 * rank + 10 + i)
                                    for i in range(n_total)])).to(dev)
    h = torch.empty((T, H), dtype=torch.float32, device=dev)

    # prefill (reads at the stored rate: target = kmax)
    hp = torch.from_numpy(initial_stream(shape, Tp, step=1_000_000 * rank)).to(dev)
    tg_store = torch.tensor([float(shape.kmax)], dtype=torch.float64, device=dev)
    hp_work = hp.clone()
    stack.forward(hp_work, tg_store, bufs)          # warm-up (module load, attributes)
    torch.cuda.synchronize()
    hp_work.copy_(hp)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    stack.forward(hp_work, tg_store, bufs)
    e1.record()
    torch.cuda.synchronize()
    prefill_ms = e0.elapsed_time(e1)
    assert dpa.device_status(bufs["ws"]) == 0

    # decode: one graph per budget, each one step through all layers
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    h.copy_(h0[0])
    stack.forward(h, tgs[0], small)
    torch.cuda.synchronize()
    graphs = []
    with torch.cuda.stream(s):
        for tg in tgs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                stack.forward(h, tg, small)
            graphs.append(g)
    torch.cuda.synchronize()
    nt = len(tgs)
    for i in range(args.warmup):
        h.copy_(h0[i])
        graphs[i % nt].replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record()
        for j in range(args.steps):
            h.copy_(h0[args.warmup + j])
            graphs[(args.warmup + j) % nt].replay()
        t1.record()
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    assert dpa.device_status(bufs["ws"]) == 0
    ms, prefill_ms = max_over_ranks(dist, [ms, prefill_ms], dev)
    del graphs
    n_layers = stack.n_layers
    return {"ms": ms, "prefill_ms": prefill_ms, "clocks": clk.summary(), "n_layers": n_layers,
            "build_s": build_s, "launches": args.steps * n_layers * 6 + args.steps * 1}


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_encode_job(shape, e):
    from oracle import dpa_oracle as O
    g, u, d = W.expert_weights(shape, e)
    return e, O.encode_expert(g, u, d, shape.fmt, shape.bits, shape.group)


def _encode_pool(shape, experts):
    """Oracle encode of the given experts in a spawned process pool (setup work)."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    n = max(1, min(32, (os.cpu_count() or 2) - 1, len(experts)))
    with ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as ex:
        return dict(ex.map(_oracle_encode_job, [shape] * len(experts), experts))


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_sample(shape, target, n_steps, n_pairs, seed_base=0):
    """Times the fp64 oracle (as it stands, one thread) on a bounded sample of the workload.
    Each sampled step routes and allocates its whole batch; `n_pairs` expert FFNs (dequantise at
    the pair's k, SwiGLU, down) are timed round robin over the steps' routed pairs, and their mean
    time counts once per routed pair of a step. Encoding the routed experts (offline work in the
    method too) runs beforehand in a spawned process pool and is not timed."""
    from threadpoolctl import threadpool_limits
    from oracle import dpa_oracle as O
    T, K = shape.tokens, shape.top_k
    wr = W.router_weights(shape)
    xs = [W.tokens(shape, T, step=seed_base + i) for i in range(n_steps)]
    routes = [O.route(x, wr, K, shape.norm_topk) for x in xs]
    need = sorted({int(e) for rt in routes for e in np.unique(rt[0])})
    experts = _encode_pool(shape, need)          # offline setup, not timed
    ffn_s = []
    ra_s = []
    with threadpool_limits(1):
        r = np.full((shape.n_experts, shape.bits), np.nan)
        for e, enc in experts.items():
            r[e] = enc["r"]
        per_step = max(1, -(-n_pairs // n_steps))
        for i, x in enumerate(xs):
            t0 = time.perf_counter()
            idx, g, _ = O.route(x, wr, K, shape.norm_topk)
            k, lam = O.allocate(idx, g, r, shape.kmin, shape.kmax, target)
            ra_s.append(time.perf_counter() - t0)
            xf = O.bf16_bits_to_f64(x)
            for q in range(per_step):
                p = (i * per_step + q) % (T * K)
                t, j = divmod(p, K)
                t1 = time.perf_counter()
                e, kk = int(idx[t, j]), int(k[t, j])
                wg, wu, wd = O.dequant_expert(experts[e], shape.fmt, shape.bits, kk, shape.group)
                O.expert_ffn(xf[t], wg, wu, wd)
                ffn_s.append(time.perf_counter() - t1)
    step_s = statistics.mean(ra_s) + T * K * statistics.mean(ffn_s)
    try:
        affinity = len(os.sched_getaffinity(0))
    except AttributeError:
        affinity = os.cpu_count()
    return {"value": T / step_s, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n_steps} steps of {T} token(s): route + allocate of the whole batch timed per step; "
                      f"{len(ffn_s)} of the steps' {T * K}-pair expert FFNs timed, their mean counted once per "
                      f"routed pair; fp64 numpy, 1 thread",
            "affinity_cores": affinity, "cpu_model": _cpu_model(), "ms_per_step": 1e3 * step_s,
            "seconds": sum(ra_s) + sum(ffn_s)}


# ----------------------------------------------------------------------------- main

def main(argv=None):
    args = parse_args(argv)
    shape = W.shape_by_name(args.workload)
    target = args.target if args.target is not None else headline_target(shape)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    metric = "MoE-layer decode tokens/s at target bpw; HBM GB/s of planes read vs peak"
    config = {"workload": shape.name, "hidden": shape.hidden, "inter": shape.inter, "experts": shape.n_experts,
              "top_k": shape.top_k, "tokens_per_step": shape.tokens, "target_bpw": target,
              "format": "uniform" if shape.fmt == W.FMT_UNIFORM else "bcq", "bits": shape.bits,
              "kmin": shape.kmin, "kmax": shape.kmax, "group": shape.group, "parallelism": f"replicas{args.gpus}",
              "l2": f"inputs larger than L2: {args.copies} device copies of the layer rotated per step"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        steps = args.steps
        # a bounded sample: at most 8 steps and 4 expert FFNs per step, whatever K and W are
        n_steps = max(1, min(8, args.warmup + steps))
        smp = oracle_sample(shape, target, n_steps, 4 * n_steps)
        line = {"impl": "reference", "metric": metric, "value": smp["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": steps, "warmup": args.warmup, "ms_per_step": smp["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {k: smp[k] for k in ("value", "unit", "cores", "kind", "sample", "affinity_cores",
                                                     "cpu_model")},
                "e2e": {"value": smp["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    else:
        torch.cuda.set_device(0)

    if shape.layers > 1:
        res = run_stack(args, shape, rank, world, dist)
        secs = res["ms"] * 1e-3
        tokens = world * shape.tokens * args.steps
        config.update({"layers": res["n_layers"], "prefill_tokens": W.STACK_PREFILL_TOKENS,
                       "target_bpw": "cycled", "targets_cycled": list(shape.targets),
                       "l2": "48 resident layers (~15 GB) per step, far larger than L2"})
        line = {"metric": metric, "value": tokens / secs, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms"] / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "u8s8-i32/f32 (decision path f64)", "data": "synthetic", "config": config,
                "prefill_tokens_per_s": world * W.STACK_PREFILL_TOKENS / (res["prefill_ms"] * 1e-3),
                "prefill_ms": res["prefill_ms"], "clocks": res["clocks"], "gpu_launches": res["launches"],
                "host_build_s": res["build_s"]}
        # whole-prefill tensor throughput: 2 flop per multiply-add of the three expert matrices over
        # every routed pair and layer (routing, allocation and glue counted in the time, not the flops)
        flops = 2.0 * W.STACK_PREFILL_TOKENS * shape.top_k * 3 * shape.hidden * shape.inter * res["n_layers"]
        pk = _peaks()
        peak = pk.get("bf16_tflops_sustained") if pk else None
        achieved = flops / (res["prefill_ms"] * 1e-3) / 1e12
        line["prefill_roofline"] = {"bound": "tensor", "achieved": achieved,
                                    "peak": peak if peak else FALLBACK_BF16_TFLOPS, "unit": "TFLOP/s",
                                    "frac": achieved / (peak if peak else FALLBACK_BF16_TFLOPS),
                                    "scope": "whole prefill step (route, allocate, permute, GEMMs, combine, glue)",
                                    "peak_source": "measured sustained bf16" if peak else "fallback"}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    if args.offload:
        res = run_offload(args, shape, target, rank, world, dist)
        pre = res["prefix"]
        config.update({"offload": "experts in pinned host memory; each step streams the first kmax_e planes of "
                                  "its routed experts host->device before the layer runs",
                       "l2": "weights streamed from host memory every step"})
        line = {"metric": metric, "value": pre["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": pre["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "u8s8-i32/f32 (decision path f64)", "data": "synthetic", "config": config,
                "h2d_bytes_per_step": pre["h2d_bytes_per_step"], "h2d_gbs": pre["h2d_gbs"],
                "full_width_streaming": res["full"],
                "gpu_launches": args.steps * ((1 if shape.tokens < 128 else 3) + 1 + 1 + 6)}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    targets = [target]
    if args.target is None and not args.no_sweep and len(shape.targets) > 1:
        targets += [t for t in shape.targets if t != target]
    results = run_dpa(args, shape, targets, rank, world, dist)
    hbm, peak_kind = peaks()
    tokens = world * shape.tokens * args.steps

    def summarise(res):
        stage = res["stage_ms"]
        dominant = max(("gateup", "down"), key=lambda n: stage[n])
        dom_bytes = res["gu_bytes"] if dominant == "gateup" else res["dn_bytes"]
        dom_s = stage[dominant] * 1e-3
        achieved = dom_bytes / dom_s / 1e9 if dom_s > 0 else 0.0
        all_bytes = res["gu_bytes"] + res["dn_bytes"]
        secs = res["ms"] * 1e-3
        gu_s, dn_s = stage["gateup"] * 1e-3, stage["down"] * 1e-3
        return dominant, achieved, all_bytes, secs, {
            "target_bpw": res["target"], "value": tokens / secs, "ms_per_step": res["ms"] / args.steps,
            "mean_planes_per_pair": res["mean_bpw"], "bytes_per_step": all_bytes / args.steps,
            "active_experts_per_step": res["n_active"] / args.steps,
            "gateup_gbs": res["gu_bytes"] / gu_s / 1e9 if gu_s > 0 else None,
            "gateup_frac": res["gu_bytes"] / gu_s / 1e9 / hbm if gu_s > 0 else None,
            "down_gbs": res["dn_bytes"] / dn_s / 1e9 if dn_s > 0 else None,
            "down_frac": res["dn_bytes"] / dn_s / 1e9 / hbm if dn_s > 0 else None,
            "planes_frac_whole_step": all_bytes / secs / 1e9 / world / hbm,
            "clocks": res["clocks"]}

    res = results[0]
    dominant, achieved, all_bytes, secs, head = summarise(res)
    stage = res["stage_ms"]
    line = {
        "metric": metric,
        "value": tokens / secs,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": res["ms"] / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8s8-i32/f32 (decision path f64)",
        "data": "synthetic",
        "config": config,
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": NCU_TRAFFIC_BYTES.get((shape.name, target)),
                     "traffic_unit": "bytes per launch", "peak_source": peak_kind},
        "planes_gbs_whole_step": all_bytes / secs / 1e9 / world,
        "planes_frac_whole_step": all_bytes / secs / 1e9 / world / hbm,
        "bytes_per_step": all_bytes / args.steps,
        "active_experts_per_step": res["n_active"] / args.steps,
        "mean_planes_per_pair": res["mean_bpw"],
        "stages_us_per_step": {k: 1e3 * v / args.steps for k, v in stage.items()},
        "clocks": res["clocks"],
        "e2e": res["e2e"],
        "gpu_launches": res["launches"],
    }
    if len(results) > 1:
        line["sweep"] = [summarise(r_)[4] for r_ in results]
    if res["tc"]:
        # prefill-sized batches run the expert FFN as tcgen05 GEMMs: tensor-bound. The gate/up stage
        # (row permutation + GEMM) is timed against the sustained bf16 peak (it runs inside a step).
        pk = _peaks()
        tpeak = pk.get("bf16_tflops_sustained") or FALLBACK_BF16_TFLOPS
        flops = 2.0 * shape.tokens * shape.top_k * 2 * shape.hidden * shape.inter * args.steps
        gu_s = stage["gateup"] * 1e-3
        ach = flops / gu_s / 1e12 if gu_s > 0 else 0.0
        line["roofline"] = {"bound": "tensor", "kernel": "gateup", "achieved": ach, "peak": tpeak,
                            "unit": "TFLOP/s", "frac": ach / tpeak,
                            "traffic": NCU_TRAFFIC_BYTES.get((shape.name, target)), "traffic_unit": "bytes per launch",
                            "peak_source": "measured sustained bf16" if pk.get("bf16_tflops_sustained") else "fallback"}
        line["dtype"] = "bf16/fp16 tensor-core operands, f32 accumulate (decision path f64)"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        smp = oracle_sample(shape, target, 4, args.cpu_sample_pairs, seed_base=50000)
        line["cpu_baseline"] = {k: smp[k] for k in ("value", "unit", "cores", "kind", "sample", "affinity_cores",
                                                    "cpu_model")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
