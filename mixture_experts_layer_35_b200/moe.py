"""ctypes binding of libmoe.so (declared in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch supplies device memory and the current CUDA stream.  If the library has not
been built, importing this module raises -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(6)
SCORE = {"softmax": 0, "sigmoid": 1}
ACT = {"swiglu": 0, "relu2": 1}
PATH = {"auto": 0, "small": 1, "large": 2}
SCHEDULE = {"auto": 0, "static": 1, "dynamic": 2}  # moe_sched_t
DT_BF16, DT_FP32 = 0, 1
DEVERR_BAD_EXPERT_ID, DEVERR_WAIT_TIMEOUT, DEVERR_BAD_INDEX, DEVERR_ROUTER_BOUND = 0x1, 0x2, 0x4, 0x8
WS_TOPK_IDS, WS_TOPK_W, WS_OFFSETS, WS_PERM = range(4)

# Every symbol include/moe.h declares.
EXPORTS = ("moe_router_topk", "moe_permute_workspace_size", "moe_permute", "moe_workspace_size",
           "moe_select_path", "moe_fused_forward", "moe_fused_forward_launches", "moe_fused_forward_plan",
           "moe_token_tiles", "moe_trace_size",
           "moe_workspace_region", "moe_fused_forward_timed", "moe_fused_forward_noalloc",
           "moe_noalloc_get_error", "moe_get_error", "moe_status_string")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_35_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _ci, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


class LayerDesc(ctypes.Structure):
    """Mirror of moe_layer_desc."""
    _fields_ = [(n, _ci) for n in ("T", "H", "I", "E", "top_k", "act", "score", "renorm", "I_shared", "path")] + [
        ("router_w", _vp), ("router_logits", _vp), ("bias", _vp), ("w13", _vp), ("w2", _vp),
        ("ws13", _vp), ("ws2", _vp), ("routed_scale", ctypes.c_float), ("shared_gate_w", _vp),
        ("shared_out", _vp), ("trace", _vp), ("schedule", _ci), ("fc1_tile_rows", _ci), ("fc2_tile_rows", _ci)]


_lib.moe_router_topk.argtypes = [_vp, _ci, _ci, _ci, _ci, _ci, _vp, _ci, _vp, _vp, _vp, _vp]
_lib.moe_router_topk.restype = _ci
_lib.moe_permute_workspace_size.argtypes = [_ci, _ci, _ci]
_lib.moe_permute_workspace_size.restype = _sz
_lib.moe_permute.argtypes = [_vp, _ci, _ci, _ci, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.moe_permute.restype = _ci
_lib.moe_workspace_size.argtypes = [ctypes.POINTER(LayerDesc)]
_lib.moe_workspace_size.restype = _sz
_lib.moe_select_path.argtypes = [ctypes.POINTER(LayerDesc)]
_lib.moe_select_path.restype = _ci
_lib.moe_fused_forward_launches.argtypes = [ctypes.POINTER(LayerDesc)]
_lib.moe_fused_forward_launches.restype = _ci
_lib.moe_fused_forward_plan.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(_ci), _ci]
_lib.moe_fused_forward_plan.restype = _ci
KERNEL_NAMES = ("prep", "router", "route", "topk", "refine", "select", "permute", "fc1", "fc2", "finalize")
_lib.moe_trace_size.argtypes = []
_lib.moe_trace_size.restype = _sz
TRACE_FIELDS, TRACE_MAX_CTAS = 8, 1024
TRACE_KERNELS = ("router", "fc1", "fc2")
_lib.moe_token_tiles.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(_ci), ctypes.POINTER(_ci)]
_lib.moe_token_tiles.restype = _ci
_lib.moe_workspace_region.argtypes = [ctypes.POINTER(LayerDesc), _ci, ctypes.POINTER(_sz), ctypes.POINTER(_sz)]
_lib.moe_workspace_region.restype = _ci
_lib.moe_fused_forward.argtypes = [ctypes.POINTER(LayerDesc), _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.moe_fused_forward.restype = _ci
_lib.moe_fused_forward_timed.argtypes = [ctypes.POINTER(LayerDesc), _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                                         ctypes.POINTER(_vp), _ci]
_lib.moe_fused_forward_timed.restype = _ci
_lib.moe_fused_forward_noalloc.argtypes = [ctypes.POINTER(LayerDesc), _vp, _vp, _vp, _vp, _vp, _vp]
_lib.moe_fused_forward_noalloc.restype = _ci
NOALLOC_SCRATCH_BYTES = 16 << 20  # MOE_NOALLOC_SCRATCH_BYTES
_lib.moe_noalloc_get_error.argtypes = [ctypes.POINTER(_ci), _vp]
_lib.moe_noalloc_get_error.restype = _ci
_lib.moe_get_error.argtypes = [_vp, ctypes.POINTER(_ci), _vp]
_lib.moe_get_error.restype = _ci
_lib.moe_status_string.argtypes = [_ci]
_lib.moe_status_string.restype = ctypes.c_char_p


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib():
    return _lib


def status_string(s: int) -> str:
    return _lib.moe_status_string(s).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoEError(st, where)


def router_topk(logits: torch.Tensor, top_k: int, score: str = "sigmoid", bias: Optional[torch.Tensor] = None,
                renorm: bool = True, stream=None, out=None):
    """Router top-k on [M, E] BF16 or FP32 device logits -> (weights f32, ids i32, src i32).
    ``out``: optional preallocated (weights, ids, src) tensors of shape [M, top_k]."""
    M, E = logits.shape
    dev = logits.device
    if out is not None:
        w, ids, src = out
    else:
        w = torch.empty((M, top_k), dtype=torch.float32, device=dev)
        ids = torch.empty((M, top_k), dtype=torch.int32, device=dev)
        src = torch.empty((M, top_k), dtype=torch.int32, device=dev)
    dt = DT_BF16 if logits.dtype == torch.bfloat16 else DT_FP32
    st = _lib.moe_router_topk(_ptr(logits), dt, M, E, top_k, SCORE[score], _ptr(bias), int(renorm),
                              _ptr(w), _ptr(ids), _ptr(src), _stream(stream))
    _check(st, "moe_router_topk")
    return w, ids, src


def permute_workspace_size(M: int, K: int, E: int) -> int:
    return _lib.moe_permute_workspace_size(M, K, E)


def permute(ids: torch.Tensor, E: int, ws: Optional[torch.Tensor] = None, stream=None):
    """[M, K] int32 expert ids -> (offsets [E+1], perm [M*K], inv [M*K]) int32."""
    M, K = ids.shape
    dev = ids.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(M * K, dtype=torch.int32, device=dev)
    inv = torch.empty(M * K, dtype=torch.int32, device=dev)
    if ws is None:
        ws = torch.zeros(permute_workspace_size(M, K, E), dtype=torch.uint8, device=dev)
    st = _lib.moe_permute(_ptr(ids), M, K, E, _ptr(offsets), _ptr(perm), _ptr(inv), _ptr(ws), ws.numel(),
                          _stream(stream))
    _check(st, "moe_permute")
    return offsets, perm, inv


def get_error(ws: torch.Tensor, stream=None) -> int:
    code = _ci(0)
    st = _lib.moe_get_error(_ptr(ws), ctypes.byref(code), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoEError(st, "moe_get_error")
    return code.value


def noalloc_get_error(stream=None) -> int:
    """Read and clear the error word of the static scratch (moe_noalloc_get_error)."""
    code = _ci(0)
    st = _lib.moe_noalloc_get_error(ctypes.byref(code), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoEError(st, "moe_noalloc_get_error")
    return code.value


def make_desc(T: int, H: int, I: int, E: int, top_k: int, act: str, score: str, renorm: bool, I_shared: int,
              path: str = "auto", router_w=None, router_logits=None, bias=None, w13=None, w2=None, ws13=None,
              ws2=None, routed_scale: float = 0.0, shared_gate_w=None, shared_out=None, trace=None,
              schedule: str = "auto", tiles=(0, 0)) -> LayerDesc:
    d = LayerDesc()
    d.T, d.H, d.I, d.E, d.top_k = T, H, I, E, top_k
    d.act, d.score, d.renorm, d.I_shared, d.path = ACT[act], SCORE[score], int(renorm), I_shared, PATH[path]
    d.router_w, d.router_logits, d.bias = _ptr(router_w), _ptr(router_logits), _ptr(bias)
    d.w13, d.w2, d.ws13, d.ws2 = _ptr(w13), _ptr(w2), _ptr(ws13), _ptr(ws2)
    d.routed_scale, d.shared_gate_w, d.shared_out = routed_scale, _ptr(shared_gate_w), _ptr(shared_out)
    d.trace = _ptr(trace)
    d.schedule = SCHEDULE[schedule]
    d.fc1_tile_rows, d.fc2_tile_rows = tiles
    return d


def workspace_size(desc: LayerDesc) -> int:
    return _lib.moe_workspace_size(ctypes.byref(desc))


def select_path(desc: LayerDesc) -> str:
    p = _lib.moe_select_path(ctypes.byref(desc))
    return {1: "small", 2: "large"}.get(p, "invalid")


def launches(desc: LayerDesc) -> int:
    return _lib.moe_fused_forward_launches(ctypes.byref(desc))


def kernel_plan(desc: LayerDesc):
    """Names of the kernels moe_fused_forward launches for this description, in order."""
    buf = (_ci * 16)()
    n = _lib.moe_fused_forward_plan(ctypes.byref(desc), buf, 16)
    return [KERNEL_NAMES[buf[i]] for i in range(n)]


def trace_buffer(device) -> torch.Tensor:
    """A zeroed phase-trace buffer for LayerDesc.trace (moe_trace_size bytes)."""
    n = _lib.moe_trace_size() // 8
    return torch.zeros(n, dtype=torch.int64, device=device)


def trace_summary(trace: torch.Tensor, grid: int) -> dict:
    """Per traced kernel, from the CTAs' %globaltimer stamps (microseconds): launch skew
    (last CTA entry - first), median wait for inputs (ready - entry), median load span
    (last load issued - ready), the tail (last exit - first exit), the whole kernel (last
    exit - first entry), and the spread of work units per CTA."""
    t = trace.view(len(TRACE_KERNELS), TRACE_MAX_CTAS, TRACE_FIELDS)[:, :grid].to("cpu").numpy()
    out = {}
    for k, name in enumerate(TRACE_KERNELS):
        r = t[k]
        live = r[:, 0] > 0
        if not live.any():
            continue
        r = r[live].astype("float64")
        entry, ready, loads, stores, exit_, units = (r[:, i] for i in range(6))
        med = lambda v: float(sorted(v)[len(v) // 2])  # noqa: E731
        out[name] = {"ctas": int(live.sum()),
                     "launch_skew_us": (entry.max() - entry.min()) / 1e3,
                     "input_wait_us_median": med(ready - entry) / 1e3,
                     "load_span_us_median": med(loads - ready) / 1e3,
                     "tail_us": (exit_.max() - exit_.min()) / 1e3,
                     "kernel_us": (exit_.max() - entry.min()) / 1e3,
                     "units_min_max": [int(units.min()), int(units.max())]}
    return out


def token_tiles(desc: LayerDesc):
    """(FC1, FC2) token rows per grouped-GEMM tile for this description."""
    a, b = _ci(0), _ci(0)
    _check(_lib.moe_token_tiles(ctypes.byref(desc), ctypes.byref(a), ctypes.byref(b)), "moe_token_tiles")
    return a.value, b.value


def workspace_view(desc: LayerDesc, ws: torch.Tensor, region: int, dtype=torch.int32) -> torch.Tensor:
    """A view of one intermediate kept in the workspace (moe_workspace_region)."""
    off, nb = _sz(0), _sz(0)
    _check(_lib.moe_workspace_region(ctypes.byref(desc), region, ctypes.byref(off), ctypes.byref(nb)),
           "moe_workspace_region")
    return ws[off.value:off.value + nb.value].view(dtype)


def fused_forward_raw(desc: LayerDesc, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
                      topk_w: Optional[torch.Tensor] = None, topk_ids: Optional[torch.Tensor] = None,
                      logits: Optional[torch.Tensor] = None, stream=None):
    st = _lib.moe_fused_forward(ctypes.byref(desc), _ptr(x), _ptr(out), _ptr(topk_w), _ptr(topk_ids),
                                _ptr(logits), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "moe_fused_forward")


def fused_forward_timed(desc: LayerDesc, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, events,
                        stream=None):
    """moe_fused_forward recording events[i] before kernel i and events[-1] after the last."""
    arr = (_vp * len(events))(*[e.cuda_event for e in events])
    st = _lib.moe_fused_forward_timed(ctypes.byref(desc), _ptr(x), _ptr(out), None, None, None, _ptr(ws),
                                      ws.numel(), _stream(stream), arr, len(events))
    _check(st, "moe_fused_forward_timed")


def fused_forward_noalloc(desc: LayerDesc, x: torch.Tensor, out: torch.Tensor,
                          topk_w: Optional[torch.Tensor] = None, topk_ids: Optional[torch.Tensor] = None,
                          logits: Optional[torch.Tensor] = None, stream=None):
    """moe_fused_forward_noalloc: no workspace argument; the library's static scratch is used."""
    st = _lib.moe_fused_forward_noalloc(ctypes.byref(desc), _ptr(x), _ptr(out), _ptr(topk_w), _ptr(topk_ids),
                                        _ptr(logits), _stream(stream))
    _check(st, "moe_fused_forward_noalloc")


class MoELayer:
    """A layer whose weights live on the device; ``forward`` enqueues moe_fused_forward."""

    def __init__(self, shape, weights: dict, path: str = "auto", routed_scale: float = 0.0,
                 schedule: str = "auto", tiles=(0, 0)):
        """``weights``: router_w, bias, w13, w2, and optionally ws13 / ws2 (internal shared
        expert) and shared_gate (its [H] gate row).  ``routed_scale``: 0 = none.
        ``schedule``: the grouped GEMMs' tile schedule (auto, static, dynamic).
        ``tiles``: (FC1, FC2) token rows per GEMM tile, 0 = the library's choice."""
        self.shape = shape
        self.w = weights
        self.path = path
        self.routed_scale = routed_scale
        self.schedule = schedule
        self.tiles = tuple(tiles)
        self._ws = None

    def desc(self, T: int, router_logits: Optional[torch.Tensor] = None,
             shared_out: Optional[torch.Tensor] = None, trace: Optional[torch.Tensor] = None) -> LayerDesc:
        s, w = self.shape, self.w
        Is = s.I_shared if w.get("ws13") is not None else 0
        return make_desc(T, s.H, s.I, s.E, s.K, s.act, s.score, s.renorm, Is, self.path,
                         router_w=w.get("router_w"), router_logits=router_logits, bias=w.get("bias"),
                         w13=w["w13"], w2=w["w2"], ws13=w.get("ws13"), ws2=w.get("ws2"),
                         routed_scale=self.routed_scale, shared_gate_w=w.get("shared_gate"), shared_out=shared_out,
                         trace=trace, schedule=self.schedule, tiles=self.tiles)

    def workspace(self, desc: LayerDesc, device) -> torch.Tensor:
        need = workspace_size(desc)
        if need == 0:
            raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(need, dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, x: torch.Tensor, router_logits: Optional[torch.Tensor] = None, out=None,
                return_routing: bool = False, stream=None, shared_out: Optional[torch.Tensor] = None,
                trace: Optional[torch.Tensor] = None):
        """``shared_out``: a [T, H] BF16 shared-expert output to add (no internal shared
        expert); ``out`` may be that same tensor (in-place form).  ``trace``: an optional
        phase-trace buffer (``trace_buffer``)."""
        T = x.shape[0]
        d = self.desc(T, router_logits, shared_out, trace)
        ws = self.workspace(d, x.device)
        if out is None:
            out = torch.empty((T, self.shape.H), dtype=torch.bfloat16, device=x.device)
        tw = ti = lg = None
        if return_routing:
            tw = torch.empty((T, self.shape.K), dtype=torch.float32, device=x.device)
            ti = torch.empty((T, self.shape.K), dtype=torch.int32, device=x.device)
            lg = torch.empty((T, self.shape.E), dtype=torch.float32, device=x.device)
        fused_forward_raw(d, x, out, ws, tw, ti, lg, stream)
        if return_routing:
            return out, tw, ti, lg
        return out
