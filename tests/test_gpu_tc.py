"""Tensor-core (tcgen05) prefill path against the fp64 oracle.

The decisions (top-k, gates, plane counts, lambda) come from the same kernels as on the GEMV
path and stay bit-identical; the expert FFN runs as grouped GEMMs with exact bf16/fp16 weight
operands, fp32 accumulation and an fp16 SwiGLU intermediate, and must stay within
|y - y_ref| <= 2e-3 * (1 + |y_ref|). Cases span several token tiles per expert (ragged last
tiles), mixed plane counts within an expert, and a single token."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from dynamic_any_precision_b200 import dpa, workloads as W  # noqa: E402
from oracle_jobs import reference_layer_parallel  # noqa: E402
from test_gpu_parity import GpuLayer, check_forward, within_tol  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 37, 300, 700])
@pytest.mark.parametrize("target", [2.0, 2.5, 4.0])
def test_tc_tiny_matches_oracle(T, target):
    # 8 experts, top-2: T = 700 gives ~175 pairs per expert, i.e. a full 128-token tile and a
    # ragged one, split further by plane count at fractional targets
    x = W.tokens(W.TINY, T, step=1000 + T)
    pairs = [(0, 0), (T - 1, 1), (T // 2, 0)]
    check_forward(W.TINY, x, target, sample_pairs=pairs, path=dpa.PATH_TC)


@pytest.mark.parametrize("target", [3.0, 4.0])
def test_tc_qwen3_prefill_sampled(target):
    # 256 tokens x top-8 over 128 experts: ~16 tokens per expert, mixed k at target 3.0
    x = W.tokens(W.QWEN3_B64, 256, step=7)
    check_forward(W.QWEN3_B64, x, target, token_subset=[0, 17, 128, 255], path=dpa.PATH_TC,
                  sample_pairs=[(0, 0), (17, 3), (255, 7)])


@pytest.mark.parametrize("target", [4.0, 3.0])
def test_tc_full_prefill_against_oracle(target):
    # 2048 tokens (16,384 pairs, ~128 per expert: full 128-token tiles): the oracle routes and
    # allocates every token (lambda couples the whole batch) and runs the expert FFNs of a strided
    # 64-token subset; decisions bit-identical, outputs and per-pair outputs within 2e-3
    gl = GpuLayer.get(W.QWEN3_B64)
    T = 2048
    x = W.tokens(W.QWEN3_B64, T, step=11)
    ws = dpa.new_workspace(gl.desc, T)
    y, aux, _ = gl.forward(x, target, ws=ws, with_pairs=True, path=dpa.PATH_TC)
    subset = list(range(5, T, 32))
    y_ref, ref = reference_layer_parallel(W.QWEN3_B64, x, target, subset)
    assert np.array_equal(aux["topk_idx"], ref["idx"])
    assert np.array_equal(aux["topk_gate"], ref["gates"])
    assert np.array_equal(aux["k"].astype(np.int64), ref["k"])
    assert aux["lambda"][0] == ref["lambda"]
    if target < 4.0:
        assert len(np.unique(aux["k"])) > 1
    ok, worst = within_tol(y[subset], y_ref[subset], bf16_out=True)
    assert ok, f"output tolerance exceeded: worst err/bound = {worst}"
    for (t, j), o in ref["pair_out"].items():
        ok, worst = within_tol(aux["pair_out"][t, j].astype(np.float64), o)
        assert ok, (t, j, worst)


def test_tc_agrees_with_gemv_at_full_prefill_size():
    # 2048 tokens (16,384 pairs, ~128 per expert): both CUDA paths make the same decisions and
    # their outputs agree within the tolerance each keeps against the exact result
    gl = GpuLayer.get(W.QWEN3_B64)
    x = W.tokens(W.QWEN3_B64, 2048, step=11)
    ws = dpa.new_workspace(gl.desc, 2048)
    y_tc, a_tc, _ = gl.forward(x, 4.0, ws=ws, with_pairs=False, path=dpa.PATH_TC)
    y_gv, a_gv, _ = gl.forward(x, 4.0, ws=ws, with_pairs=False, path=dpa.PATH_GEMV)
    for key in ("topk_idx", "topk_gate", "k", "lambda"):
        assert np.array_equal(a_tc[key], a_gv[key]), key
    ok, worst = within_tol(y_tc, y_gv, 4e-3)
    assert ok, worst


def test_tc_rejects_unqualified_shapes():
    # binary-coded planes have no tensor-core path
    gl = GpuLayer.get(W.DEEPSEEK_B16)
    x = W.tokens(W.DEEPSEEK_B16)
    with pytest.raises(dpa.DpaError, match="UNSUPPORTED"):
        gl.forward(x, 2.0, path=dpa.PATH_TC)
