"""The C-ABI library loads without a GPU, exports every symbol include/dpa.h declares, and
rejects bad host arguments before launching anything. CPU only."""
import ctypes
import os
import re

import numpy as np
import pytest

from dynamic_any_precision_b200 import dpa, workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(dpa_[a-z_0-9]+)\s*\(", txt))
    return names


def test_library_exports_every_declared_symbol():
    lib = dpa.lib()
    syms = declared_symbols()
    assert {"dpa_encode", "dpa_route", "dpa_allocate", "dpa_moe_forward"} <= syms
    for s in sorted(syms):
        assert hasattr(lib, s), s
    assert lib.dpa_version() >= 100
    assert lib.dpa_status_string(0) == b"ok"


def test_encoded_sizes_formula():
    for sh in W.ALL_SHAPES:
        d = dpa.make_desc(sh)
        s = dpa.encoded_sizes(d)
        H, I, B, G, E = sh.hidden, sh.inter, sh.bits, sh.group, sh.n_experts
        assert s.planes_per_expert == 3 * B * H * I // 8
        assert s.planes_bytes == E * s.planes_per_expert
        if sh.fmt == W.FMT_UNIFORM:
            assert s.meta_per_expert == 4 * (2 * I * (H // G) + H * (I // G))
        else:
            assert s.meta_per_expert == 2 * B * (2 * I * (H // G) + H * (I // G))
        assert s.rtable_bytes == 8 * E * B
        assert dpa.workspace_size(d, max(1, sh.tokens)) > 0


@pytest.mark.parametrize("field,value,code", [
    ("hidden", 100, 2), ("group", 32, 2), ("bits", 5, 2), ("kmin", 0, 1), ("kmax", 5, 1),
    ("top_k", 9, 1), ("norm_topk", 2, 1), ("format", 3, 1), ("n_experts", 0, 1), ("n_experts", 2000, 2)])
def test_descriptor_validation(field, value, code):
    d = dpa.make_desc(W.TINY)
    setattr(d, field, value)
    s = dpa.Sizes()
    assert dpa.lib().dpa_encoded_sizes(ctypes.byref(d), ctypes.byref(s)) == code


@pytest.mark.parametrize("hidden,group,code", [(2048, 128, 0), (4608, 128, 0), (8192, 128, 0), (11264, 128, 0),
                                              (12288, 128, 2), (10240, 64, 2), (16384, 64, 2)])
def test_hidden_size_limit(hidden, group, code):
    # the expert GEMV keeps a token group's activation digits for every input column in shared
    # memory beside a ring of two or more plane stages: a layer is accepted while that fits
    # (group 128: hidden up to 11264)
    d = dpa.make_desc(W.with_sizes(W.QWEN3_B64, hidden=hidden, group=group, name=f"h{hidden}"))
    s = dpa.Sizes()
    assert dpa.lib().dpa_encoded_sizes(ctypes.byref(d), ctypes.byref(s)) == code


def test_host_argument_errors_launch_nothing():
    lib = dpa.lib()
    d = dpa.make_desc(W.TINY)
    buf = ctypes.c_void_p(16 * 1024)  # never dereferenced: validation fails first
    # n_tokens = 0, null pointers, misalignment, small workspace
    assert lib.dpa_route(ctypes.byref(d), buf, 0, buf, buf, buf, None, buf, 1 << 30, None) == 1
    assert lib.dpa_route(ctypes.byref(d), None, 4, buf, buf, buf, None, buf, 1 << 30, None) == 1
    assert lib.dpa_route(ctypes.byref(d), ctypes.c_void_p(16 * 1024 + 2), 4, buf, buf, buf, None, buf, 1 << 30,
                         None) == 1
    assert lib.dpa_route(ctypes.byref(d), buf, 4, buf, buf, buf, None, buf, 16, None) == 3
    assert lib.dpa_allocate(ctypes.byref(d), buf, buf, buf, 4, None, buf, None, buf, 1 << 30, None) == 1
    w = dpa.LayerWeights(16 * 1024, 16 * 1024, None, 16 * 1024, None, None, None)
    assert lib.dpa_moe_forward(ctypes.byref(d), ctypes.byref(w), buf, 4, buf, buf, None, buf, 1 << 30, None) == 1
    w = dpa.LayerWeights(16 * 1024, 16 * 1024, 16 * 1024, 16 * 1024, None, None, None)
    assert lib.dpa_moe_forward(ctypes.byref(d), ctypes.byref(w), buf, 4, buf, buf, None, buf, 64, None) == 3
    assert lib.dpa_device_status(None, None) == 1


def test_encode_rejects_bad_ranges():
    d = dpa.make_desc(W.TINY)
    g = np.zeros((1, W.TINY.inter, W.TINY.hidden), np.float32)
    dn = np.zeros((1, W.TINY.hidden, W.TINY.inter), np.float32)
    with pytest.raises(dpa.DpaError):
        dpa.encode(d, g, g, dn, e_begin=W.TINY.n_experts)      # past the last expert
    big = g.copy()
    big[0, 0, 0] = 1e9                                        # range does not fit an fp16 scale
    with pytest.raises(dpa.DpaError):
        dpa.encode(d, big, g, dn)
