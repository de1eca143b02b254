"""Host logic of bench.py on CPU: the max-over-ranks device time with two gloo ranks (the
replicas path that torchrun runs one process per GPU), the per-rank token seeds, and the
reference arm's JSON line on the tiny layer."""
import datetime
import io
import json
import os
import socket
from contextlib import redirect_stdout

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402
from dynamic_any_precision_b200 import workloads as W  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "measured" 1 + r, 10 - r and 3.5 ms: every rank must get the maxima
        got = bench.max_over_ranks(dist, [1.0 + rank, 10.0 - rank, 3.5], "cpu")
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = dict(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert results[0] == results[1] == [2.0, 10.0, 3.5]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(None, [1, 2.5], "cpu") == [1.0, 2.5]


def test_replica_token_seeds_are_distinct_per_rank_and_step():
    seeds = {bench.replica_token_seed(r, i) for r in range(8) for i in range(4096)}
    assert len(seeds) == 8 * 4096
    a = W.tokens(W.TINY, 4, step=bench.replica_token_seed(0, 3))
    b = W.tokens(W.TINY, 4, step=bench.replica_token_seed(1, 3))
    assert not (a == b).all()


def test_reference_arm_prints_one_contract_line():
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--workload", W.TINY.name, "--steps", "2", "--warmup", "0"])
    assert rc == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["config"]["workload"] == W.TINY.name
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] == 1 and line["cpu_baseline"]["affinity_cores"] >= 1
    assert isinstance(line["cpu_baseline"]["cpu_model"], str)
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_headline_budget_of_each_workload():
    # the batch-64 layer is quoted at the middle of its budget sweep, the others at their budget
    assert bench.headline_target(W.QWEN3_B64) == 3.0
    assert bench.headline_target(W.QWEN3_B1) == 2.5
    assert bench.parse_args([]).workload == W.QWEN3_B64.name
