"""Thin Python binding of the C ABI in include/dpa.h (argument marshalling only).

Device buffers are torch CUDA tensors (PyTorch provides memory and streams); every
computation runs in the CUDA library lib/libdpa_b200.so. There is no CPU fallback: if the
library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# the in-tree build; DPA_LIB may name another build of the same library (e.g. a debug build)
LIB_PATH = os.environ.get("DPA_LIB") or os.path.join(_PKG, "lib", "libdpa_b200.so")

DPA_OK = 0
STATUS_NAMES = {0: "DPA_OK", 1: "DPA_ERR_INVALID_ARG", 2: "DPA_ERR_UNSUPPORTED", 3: "DPA_ERR_WORKSPACE",
                4: "DPA_ERR_CUDA", 5: "DPA_ERR_DEVICE_TIMEOUT", 6: "DPA_ERR_DEVICE_INVALID_INPUT"}
FMT_UNIFORM, FMT_BCQ = 0, 1
MAT_GATE, MAT_UP, MAT_DOWN = 0, 1, 2


class DpaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class LayerDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("hidden", "inter", "n_experts", "top_k", "n_shared", "format", "bits", "kmin", "kmax",
                 "group", "norm_topk")]


class Sizes(ctypes.Structure):
    _fields_ = [("planes_bytes", ctypes.c_uint64), ("meta_bytes", ctypes.c_uint64),
                ("rtable_bytes", ctypes.c_uint64), ("planes_per_expert", ctypes.c_uint64),
                ("meta_per_expert", ctypes.c_uint64), ("planes_matrix_offset", ctypes.c_uint64 * 3),
                ("meta_matrix_offset", ctypes.c_uint64 * 3)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("planes", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("rtable", ctypes.c_void_p),
                ("w_router", ctypes.c_void_p), ("shared_gate", ctypes.c_void_p),
                ("shared_up", ctypes.c_void_p), ("shared_down", ctypes.c_void_p),
                ("expert_width", ctypes.c_void_p), ("expert_offsets", ctypes.c_void_p)]


class Aux(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_gate", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("lambda_", ctypes.c_void_p), ("pair_out", ctypes.c_void_p),
                ("events", ctypes.c_void_p * 7), ("expert_path", ctypes.c_int32),
                ("alloc_policy", ctypes.c_int32), ("threshold", ctypes.c_void_p), ("expert_k", ctypes.c_void_p)]

PATH_AUTO, PATH_GEMV, PATH_TC = 0, 1, 2
ALLOC_LAGRANGE, ALLOC_UNIFORM, ALLOC_THRESHOLD, ALLOC_EXPERT_TABLE = 0, 1, 2, 3


EXPORTED = ("dpa_encoded_sizes", "dpa_encode", "dpa_export_codes", "dpa_export_meta", "dpa_route",
            "dpa_allocate", "dpa_allocate_ex", "dpa_calibrate_threshold", "dpa_forward_workspace_size",
            "dpa_moe_forward", "dpa_device_status", "dpa_status_string", "dpa_version", "dpa_residual_rmsnorm",
            "dpa_debug_timeout_probe", "dpa_distortion_tensor", "dpa_profile_prefill", "dpa_solve_expert_rates",
            "dpa_stream_prefixes", "dpa_solve_stored_widths", "dpa_compact_sizes", "dpa_compact_layer")

_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run `python -m dynamic_any_precision_b200.build`)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    P = ctypes.POINTER
    L.dpa_encoded_sizes.argtypes = [P(LayerDesc), P(Sizes)]
    L.dpa_encode.argtypes = [P(LayerDesc), i32, i32, vp, vp, vp, vp, vp, vp, i32]
    L.dpa_export_codes.argtypes = [P(LayerDesc), vp, i32, i32, vp]
    L.dpa_export_meta.argtypes = [P(LayerDesc), vp, i32, i32, vp, vp]
    L.dpa_route.argtypes = [P(LayerDesc), vp, i32, vp, vp, vp, vp, vp, sz, vp]
    L.dpa_allocate.argtypes = [P(LayerDesc), vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]
    L.dpa_allocate_ex.argtypes = [P(LayerDesc), i32, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.dpa_distortion_tensor.argtypes = [P(LayerDesc), i32, i32, vp, vp, vp, vp, vp, i32]
    L.dpa_profile_prefill.argtypes = [P(LayerDesc), vp, i32, vp, vp, vp, vp, sz, vp]
    L.dpa_solve_expert_rates.argtypes = [P(LayerDesc), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.dpa_calibrate_threshold.argtypes = [P(LayerDesc), vp, i32, vp, vp, vp, sz, vp]
    L.dpa_forward_workspace_size.argtypes = [P(LayerDesc), i32]
    L.dpa_forward_workspace_size.restype = sz
    L.dpa_moe_forward.argtypes = [P(LayerDesc), P(LayerWeights), vp, i32, vp, vp, P(Aux), vp, sz, vp]
    L.dpa_device_status.argtypes = [vp, vp]
    L.dpa_debug_timeout_probe.argtypes = [vp, sz, i32, ctypes.c_uint64, vp]
    L.dpa_stream_prefixes.argtypes = [P(LayerDesc), vp, vp, vp, vp, i32, vp, vp, P(ctypes.c_uint64), vp]
    L.dpa_residual_rmsnorm.argtypes = [vp, vp, i32, i32, vp, vp]
    L.dpa_solve_stored_widths.argtypes = [P(LayerDesc), vp, vp, ctypes.c_int64, vp]
    L.dpa_compact_sizes.argtypes = [P(LayerDesc), vp, P(ctypes.c_uint64), P(ctypes.c_uint64)]
    L.dpa_compact_layer.argtypes = [P(LayerDesc), vp, vp, vp, vp, vp, vp]
    L.dpa_status_string.argtypes = [i32]
    L.dpa_status_string.restype = ctypes.c_char_p
    L.dpa_version.argtypes = []
    for name in EXPORTED:
        if name not in ("dpa_forward_workspace_size", "dpa_status_string", "dpa_version"):
            getattr(L, name).restype = i32
    L.dpa_version.restype = i32
    _lib = L
    return L


def _check(st: int, where: str):
    if st != DPA_OK:
        raise DpaError(st, where)


def make_desc(shape) -> LayerDesc:
    """Descriptor from a workloads.LayerShape (or any object with the same fields)."""
    return LayerDesc(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared, shape.fmt,
                     shape.bits, shape.kmin, shape.kmax, shape.group, shape.norm_topk)


def encoded_sizes(desc: LayerDesc) -> Sizes:
    s = Sizes()
    _check(lib().dpa_encoded_sizes(ctypes.byref(desc), ctypes.byref(s)), "dpa_encoded_sizes")
    return s


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def encode(desc: LayerDesc, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray, e_begin: int = 0,
           out: Optional[Tuple[np.ndarray, np.ndarray, np.ndarray]] = None, n_threads: int = 0):
    """Host encoder. w_* hold experts [e_begin, e_begin + n) as contiguous fp32 arrays.
    Returns (planes uint8, meta uint8, rtable fp64 [E][B]) for the whole layer (only the
    given experts' parts are written; pass `out` to fill buffers from earlier calls)."""
    s = encoded_sizes(desc)
    if out is None:
        planes = np.zeros(s.planes_bytes, np.uint8)
        meta = np.zeros(s.meta_bytes, np.uint8)
        rtable = np.zeros((desc.n_experts, desc.bits), np.float64)
    else:
        planes, meta, rtable = out
    wg = np.ascontiguousarray(w_gate, np.float32)
    wu = np.ascontiguousarray(w_up, np.float32)
    wd = np.ascontiguousarray(w_down, np.float32)
    n = wg.shape[0] if wg.ndim == 3 else 1
    _check(lib().dpa_encode(ctypes.byref(desc), e_begin, n, _ptr(wg), _ptr(wu), _ptr(wd), _ptr(planes), _ptr(meta),
                            _ptr(rtable), n_threads), "dpa_encode")
    return planes, meta, rtable


def export_codes(desc: LayerDesc, planes: np.ndarray, expert: int, matrix: int) -> np.ndarray:
    R = desc.hidden if matrix == MAT_DOWN else desc.inter
    C = desc.inter if matrix == MAT_DOWN else desc.hidden
    out = np.empty((R, C), np.uint8)
    _check(lib().dpa_export_codes(ctypes.byref(desc), _ptr(planes), expert, matrix, _ptr(out)), "dpa_export_codes")
    return out


def export_meta(desc: LayerDesc, meta: np.ndarray, expert: int, matrix: int):
    R = desc.hidden if matrix == MAT_DOWN else desc.inter
    C = desc.inter if matrix == MAT_DOWN else desc.hidden
    ng = C // desc.group
    if desc.format == FMT_UNIFORM:
        s = np.empty((R, ng), np.float32)
        z = np.empty((R, ng), np.float32)
        _check(lib().dpa_export_meta(ctypes.byref(desc), _ptr(meta), expert, matrix, _ptr(s), _ptr(z)),
               "dpa_export_meta")
        return s, z
    al = np.empty((desc.bits, R, ng), np.float32)
    _check(lib().dpa_export_meta(ctypes.byref(desc), _ptr(meta), expert, matrix, _ptr(al), None), "dpa_export_meta")
    return al, None


# ----------------------------------------------------------------------------- device calls

def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def workspace_size(desc: LayerDesc, max_tokens: int) -> int:
    n = lib().dpa_forward_workspace_size(ctypes.byref(desc), max_tokens)
    if n == 0:
        raise DpaError(1, "dpa_forward_workspace_size")
    return n


def new_workspace(desc: LayerDesc, max_tokens: int, device=None):
    """Zero-filled workspace (the library requires it zeroed once before first use)."""
    import torch
    return torch.zeros(workspace_size(desc, max_tokens), dtype=torch.uint8, device=device or "cuda")


def route(desc: LayerDesc, x, w_router, ws, logits=None, stream=None):
    """x: CUDA uint16/bf16 [T][H]; w_router: [E][H]. Returns (idx int32 [T][K], gate fp64 [T][K])."""
    import torch
    T = x.shape[0]
    idx = torch.empty((T, desc.top_k), dtype=torch.int32, device=x.device)
    gate = torch.empty((T, desc.top_k), dtype=torch.float64, device=x.device)
    _check(lib().dpa_route(ctypes.byref(desc), _dptr(x), T, _dptr(w_router), _dptr(idx), _dptr(gate),
                           _dptr(logits), _dptr(ws), ws.numel(), _stream(stream)), "dpa_route")
    return idx, gate


def allocate(desc: LayerDesc, rtable, idx, gate, target, ws, stream=None, policy: int = ALLOC_LAGRANGE,
             threshold=None, expert_k=None):
    """target: CUDA fp64 scalar tensor (None for the threshold and table policies); threshold:
    CUDA fp64 scalar tensor (threshold policy); expert_k: CUDA uint8 [E] (table policy).
    Returns (k uint8 [T][K], lambda fp64 [1])."""
    import torch
    T = idx.shape[0]
    k = torch.empty((T, desc.top_k), dtype=torch.uint8, device=idx.device)
    lam = torch.empty(1, dtype=torch.float64, device=idx.device)
    if policy == ALLOC_LAGRANGE:
        _check(lib().dpa_allocate(ctypes.byref(desc), _dptr(rtable), _dptr(idx), _dptr(gate), T, _dptr(target),
                                  _dptr(k), _dptr(lam), _dptr(ws), ws.numel(), _stream(stream)), "dpa_allocate")
    else:
        _check(lib().dpa_allocate_ex(ctypes.byref(desc), policy, _dptr(rtable), _dptr(idx), _dptr(gate), T,
                                     _dptr(target), _dptr(threshold), _dptr(expert_k), _dptr(k), _dptr(lam),
                                     _dptr(ws), ws.numel(), _stream(stream)), "dpa_allocate_ex")
    return k, lam


def distortion_tensor(desc: LayerDesc, w_gate: np.ndarray, w_up: np.ndarray, planes: np.ndarray, meta: np.ndarray,
                      e_begin: int = 0, out: Optional[np.ndarray] = None, n_threads: int = 0) -> np.ndarray:
    """Host distortion tensor [E][B][H] fp64 for experts [e_begin, e_begin + n) of the layer."""
    T = np.zeros((desc.n_experts, desc.bits, desc.hidden), np.float64) if out is None else out
    wg = np.ascontiguousarray(w_gate, np.float32)
    wu = np.ascontiguousarray(w_up, np.float32)
    n = wg.shape[0] if wg.ndim == 3 else 1
    _check(lib().dpa_distortion_tensor(ctypes.byref(desc), e_begin, n, _ptr(wg), _ptr(wu), _ptr(planes), _ptr(meta),
                                       _ptr(T), n_threads), "dpa_distortion_tensor")
    return T


def profile_prefill(desc: LayerDesc, x, idx, ws, stream=None):
    """x: CUDA bf16 bits [T][H]; idx: CUDA int32 [T][K]. Returns (m fp64 [H], counts int32 [E])."""
    import torch
    m = torch.empty(desc.hidden, dtype=torch.float64, device=x.device)
    counts = torch.empty(desc.n_experts, dtype=torch.int32, device=x.device)
    _check(lib().dpa_profile_prefill(ctypes.byref(desc), _dptr(x), x.shape[0], _dptr(idx), _dptr(m), _dptr(counts),
                                     _dptr(ws), ws.numel(), _stream(stream)), "dpa_profile_prefill")
    return m, counts


def solve_expert_rates(desc: LayerDesc, tdist, m, counts, target, ws, stream=None):
    """tdist: CUDA fp64 [E][B][H]. Returns (k_table uint8 [E], lambda fp64 [1])."""
    import torch
    kt = torch.empty(desc.n_experts, dtype=torch.uint8, device=m.device)
    lam = torch.empty(1, dtype=torch.float64, device=m.device)
    _check(lib().dpa_solve_expert_rates(ctypes.byref(desc), _dptr(tdist), _dptr(m), _dptr(counts), _dptr(target),
                                        _dptr(kt), _dptr(lam), _dptr(ws), ws.numel(), _stream(stream)),
           "dpa_solve_expert_rates")
    return kt, lam


def calibrate_threshold(desc: LayerDesc, scores, target, ws, stream=None):
    """scores: CUDA fp64 tensor (any shape) of calibration routing scores; target: CUDA fp64
    scalar tensor. Returns the threshold as a CUDA fp64 [1] tensor."""
    import torch
    tau = torch.empty(1, dtype=torch.float64, device=scores.device)
    _check(lib().dpa_calibrate_threshold(ctypes.byref(desc), _dptr(scores), scores.numel(), _dptr(target), _dptr(tau),
                                         _dptr(ws), ws.numel(), _stream(stream)), "dpa_calibrate_threshold")
    return tau


class DeviceLayer:
    """Encoded layer resident in device memory (torch tensors) plus its C weight struct."""

    def __init__(self, desc: LayerDesc, planes, meta, rtable, w_router, shared=None, widths=None, offsets=None):
        """widths (uint8 [E]) and offsets (uint64 [E][2] as int64) on the device: a compact layer
        of per-expert stored widths (dpa_compact_layer); both None: the full layout."""
        self.desc = desc
        self.planes, self.meta, self.rtable, self.w_router = planes, meta, rtable, w_router
        self.shared = shared
        self.widths, self.offsets = widths, offsets
        sg, su, sd = shared if shared is not None else (None, None, None)
        self.weights = LayerWeights(_dptr(planes), _dptr(meta), _dptr(rtable), _dptr(w_router), _dptr(sg),
                                    _dptr(su), _dptr(sd), _dptr(widths), _dptr(offsets))

    @classmethod
    def from_host(cls, desc: LayerDesc, planes: np.ndarray, meta: np.ndarray, rtable: np.ndarray,
                  w_router_bits: np.ndarray, shared_bits=None, device="cuda"):
        import torch

        def dev(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)
        sh = None
        if shared_bits is not None:
            sh = tuple(dev(s.view(np.int16)) for s in shared_bits)
        return cls(desc, dev(planes), dev(meta), dev(rtable), dev(w_router_bits.view(np.int16)), sh)


def moe_forward(layer: DeviceLayer, x, target, ws, y=None, aux: Optional[dict] = None, stream=None):
    """One MoE layer. x: CUDA int16/bf16 bits [T][H]; target: CUDA fp64 scalar tensor.
    aux: optional dict of preallocated CUDA tensors with keys topk_idx, topk_gate, k, lambda,
    pair_out, "events": up to 7 torch.cuda.Event(enable_timing=True) recorded at the
    stage boundaries, "expert_path" (PATH_AUTO, PATH_GEMV or PATH_TC), "alloc_policy"
    (ALLOC_LAGRANGE, ALLOC_UNIFORM or ALLOC_THRESHOLD) and "threshold" (CUDA fp64 scalar).
    Returns y (int16 bf16 bits [T][H])."""
    import torch
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, layer.desc.hidden), dtype=torch.int16, device=x.device)
    aux_s = None
    if aux:
        aux_s = Aux(_dptr(aux.get("topk_idx")), _dptr(aux.get("topk_gate")), _dptr(aux.get("k")),
                    _dptr(aux.get("lambda")), _dptr(aux.get("pair_out")))
        for i, ev in enumerate(aux.get("events") or ()):
            if ev is not None:
                if not ev.cuda_event:
                    raise ValueError("record a torch.cuda.Event once before passing it (lazy creation)")
                aux_s.events[i] = ev.cuda_event
        aux_s.expert_path = int(aux.get("expert_path", PATH_AUTO))
        aux_s.alloc_policy = int(aux.get("alloc_policy", ALLOC_LAGRANGE))
        aux_s.threshold = _dptr(aux.get("threshold"))
        aux_s.expert_k = _dptr(aux.get("expert_k"))
    _check(lib().dpa_moe_forward(ctypes.byref(layer.desc), ctypes.byref(layer.weights), _dptr(x), T, _dptr(target),
                                 _dptr(y), ctypes.byref(aux_s) if aux_s is not None else None, _dptr(ws), ws.numel(),
                                 _stream(stream)), "dpa_moe_forward")
    return y


def residual_rmsnorm(h, x, y=None, stream=None):
    """Stack glue: h += y (if given), x = bf16(RMSNorm(h)). h fp32 [T][H] (in place),
    x and y bf16 bits [T][H] (int16 tensors)."""
    T, H = h.shape
    _check(lib().dpa_residual_rmsnorm(_dptr(y), _dptr(h), T, H, _dptr(x), _stream(stream)), "dpa_residual_rmsnorm")
    return x


def stream_prefixes(desc: LayerDesc, host_planes, host_meta, experts, kplanes, dev_planes, dev_meta,
                    stream=None) -> int:
    """Copy the first kplanes[i] planes (and their scale data) of experts[i] from the host
    layer (pinned torch uint8 tensors) to the device layer. Returns the bytes issued."""
    ex = np.ascontiguousarray(experts, dtype=np.int32)
    kp = np.ascontiguousarray(kplanes, dtype=np.uint8)
    nbytes = ctypes.c_uint64(0)
    _check(lib().dpa_stream_prefixes(ctypes.byref(desc), host_planes.data_ptr(), host_meta.data_ptr(), _ptr(ex),
                                     _ptr(kp), int(ex.size), _dptr(dev_planes), _dptr(dev_meta), ctypes.byref(nbytes),
                                     _stream(stream)), "dpa_stream_prefixes")
    return int(nbytes.value)


def solve_stored_widths(desc: LayerDesc, importance: np.ndarray, rtable: np.ndarray, budget_planes: int) -> np.ndarray:
    """Per-expert stored planes (uint8 [E]) minimising sum_e importance[e] * rtable[e][b_e - 1]
    within a budget of stored planes over all experts (host)."""
    imp = np.ascontiguousarray(importance, dtype=np.float64)
    r = np.ascontiguousarray(rtable, dtype=np.float64)
    w = np.zeros(desc.n_experts, dtype=np.uint8)
    _check(lib().dpa_solve_stored_widths(ctypes.byref(desc), _ptr(imp), _ptr(r), int(budget_planes), _ptr(w)),
           "dpa_solve_stored_widths")
    return w


def compact_layer(desc: LayerDesc, planes: np.ndarray, meta: np.ndarray, widths: np.ndarray):
    """Host compact layer for per-expert stored widths: (planes, meta, offsets uint64 [E][2])."""
    w = np.ascontiguousarray(widths, dtype=np.uint8)
    pb, mb = ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check(lib().dpa_compact_sizes(ctypes.byref(desc), _ptr(w), ctypes.byref(pb), ctypes.byref(mb)),
           "dpa_compact_sizes")
    po = np.zeros(pb.value, dtype=np.uint8)
    mo = np.zeros(mb.value, dtype=np.uint8)
    off = np.zeros((desc.n_experts, 2), dtype=np.uint64)
    _check(lib().dpa_compact_layer(ctypes.byref(desc), _ptr(np.ascontiguousarray(planes)),
                                   _ptr(np.ascontiguousarray(meta)), _ptr(w), _ptr(po), _ptr(mo), _ptr(off)),
           "dpa_compact_layer")
    return po, mo, off


def device_error_detail(ws) -> Tuple[int, int]:
    """(code, detail) of the device error flag in ws, without clearing it (synchronises). The
    detail says which check or wait recorded it."""
    import torch
    torch.cuda.synchronize(ws.device)
    v = ws[:8].cpu().numpy().view(np.uint32)
    return int(v[0]), int(v[1])


def device_status(ws, stream=None) -> int:
    """Synchronise, read and clear the device error flag; returns the status code."""
    return int(lib().dpa_device_status(_dptr(ws), _stream(stream)))
